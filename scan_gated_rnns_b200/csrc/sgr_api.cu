// sgr_api.cu -- host side of the C ABI declared in include/scan_gated_rnns.h:
// argument checks, the choice of chunk shape, the workspace layout and the
// kernel launches.  No allocation, no synchronisation on the scan paths.
#include "scan_gated_rnns.h"
#include "projected_scan.cuh"
#include "scan_backward.cuh"
#include "scan_engine.cuh"
#include "scan_fold.cuh"
#include "scan_pipelined_backward.cuh"
#include "scan_sequential.cuh"

#include <algorithm>
#include <atomic>
#include <cstring>
#include <limits>
#include <mutex>
#include <utility>
#include <vector>

namespace {

using namespace sgr;

// Blocks are whole multiples of 4 warps (7 or 15 data warps + 1 carry warp),
// so they spread evenly over the SM's 4 sub-partitions, each of which has its
// own register file: 128 registers per thread with two 8-warp pipelined
// blocks or one 16-warp block per SM.
constexpr int kWarps = 7;
constexpr int kPipeWarps = 7;        // two blocks per SM
constexpr int kPipeWarpsWide = 15;   // one block per SM, tiles twice as long
constexpr int kStages = 3;
// the fp32 pipelined gradients: two blocks of 6 data warps + 1 carry warp per
// SM, 4 rows per thread, a 2-slot ring (three slots of their 96-row tiles
// would not leave room for a second block)
constexpr int kBwdPairWarps = 6;
constexpr int kBwdPairStages = 2;
constexpr int kAssumedSMs = 148;     // B200; only used to pick a tile shape
constexpr int64_t kTargetTiles = 4 * 148;  // tile kernel: prefer >= 4 tiles per SM
constexpr size_t kAlign = 256;
// Workspace header, [0, 256): the status word of the bounded waits at byte 0,
// the tile kernels' chunk ticket counter at byte 64 (its own 32-byte sector).
// Every non-empty scan plan has the header; hand-off words follow it.
constexpr size_t kTicketOffset = 64;

enum Kind { KIND_AUTO = 0, KIND_TILE = 1, KIND_PIPELINED = 2, KIND_PIPELINED_WIDE = 3, KIND_SEQUENTIAL = 4,
            KIND_SEQUENTIAL_SPLIT = 5, KIND_SEQUENTIAL_PAIR = 6, KIND_SEQUENTIAL_PAIR2 = 7, KIND_SEQUENTIAL_QUAD = 8 };
bool seq_kind(int k) {
    return k == KIND_SEQUENTIAL || k == KIND_SEQUENTIAL_SPLIT || k == KIND_SEQUENTIAL_PAIR ||
           k == KIND_SEQUENTIAL_PAIR2 || k == KIND_SEQUENTIAL_QUAD;
}

// Channel-sequential kernels (scan_sequential.cuh): each 32-channel group's
// whole sequence is walked by one warp or by a block of two warps.  Chosen
// when the groups alone give every SM at least kSeqMinWarpsPerSM of them
// (fp32) or kSeqMinWarpsPerSMHalf (bf16); below that the time axis is cut
// into chunks (measured crossovers: fp32 between 3.5 and 5.2 groups per SM,
// noisy near 5; bf16 between 3.5 and 6.9 with two warps per group).  Shared-memory
// figures are those of sm_100 (228 KB per SM, 1 KB reserved per block, 227 KB
// per block at most); the launch reads the device's own.
constexpr int kSeqMinWarpsPerSM = 6;
constexpr int kSeqMinWarpsPerSMHalf = 6;
// Below these many 32-channel groups per SM, each group takes a block of two
// warps that split every slot's rows (scan_sequential_pair_kernel): twice the
// warps hide the latency each one exposes, for a fold and a pair exchange per
// slot.  Measured on B x 2048 x D (fraction of the copy bandwidth, one warp
// per group against two): bf16 D 4096 at 6.9 groups per SM 0.53 / 0.58, 13.8:
// 0.70 / 0.76, 20.8: 0.70 / 0.75, 27.7: 0.84 / 0.76; fp32 D 2048 at 10.4:
// 0.81 / 0.84, 13.8: 0.84 / 0.86, and D 4096 at 27.7: 0.85 / 0.87.
constexpr int kSeqPairBelow = 32;
constexpr int kSeqPairBelowHalf = 24;
// From kSeqPairBelowHalf groups per SM, bf16 takes two warps per group of 64
// channels, two channels per lane (scan_sequential_pair2_kernel): the same
// warps as one per 32-channel group, fewer instructions per element.  Measured
// (us, one warp per 32 / two per 32 / two per 64 channels): B32 x 2048 x 4096
// (27.7 groups per SM) 301.6 / 315.9 / 289.2; below, the 32-channel pairs
// win: B24 (20.8) 248.3 / 238.1 / 250.4, B16 (13.8) 162.3 / 158.2 / 172.5.
// Four warps per group of 64 channels (8 rows of each slot per warp, the
// same kernel): the warps of the 32-channel pairs with the per-element work
// of the 64-channel ones.  Measured on B x 2048 x 4096 bf16 (us, two warps
// per 32 / two per 64 / four per 64 channels): minGRU B20 (17.3 groups per
// SM) 205.3 / 197.2 / 199.1, B24 238.1 / 240.1 / 231.9, B32 313.9 / 276.5 /
// 289.2; decayed B16 182.8 / 205.3 / 184.0, B20 234.0 / 248.3 / 229.3, B24
// 287.4 / 295.4 / 270.9, B28 327.1 / 334.2 / 313.9, B32 350.7 / 340.5 / 338.0;
// MinMax B8 82.5 / 76.2 / 76.5, B12 137.6 / 121.3 / 125.4, B16 156.2 / 162.3 /
// 154.1, B24 227.9 / 227.6 / 219.6, B32 309.7 / 289.2 / 277.0.  Chosen for
// bf16 MinMax wherever a channel-sequential kernel runs, and for the minGRU
// from kSeqQuadFrom groups per SM: up to kSeqPairBelowHalf for the plain
// scan (two warps per 64 channels above), throughout for the decayed one.
constexpr int kSeqQuadFrom = 16;
// The gradient (four operands in, two out per element) walks whole sequences
// from 5 warps per SM: against the pipelined gradient it loses at 3.5 groups
// per SM (bf16 B4 x 2048 x 4096 150 us against 101 us; fp32 B8 x 2048 x 2048
// a tie, its decayed form 194 against 182 us) and wins at 6.9 (bf16 B8:
// 177 against 183 us, decayed 224 against 247; fp32 B16 x 2048 x 2048 289
// against 306, decayed 308 against 349).
constexpr int kSeqBwdMinWarpsPerSM = 5;
constexpr int kSeqMaxSlots = 8;
constexpr int kSeqMinSlots = 2;
// The blocks of two or four warps per channel group keep two slots per warp
// whatever their share of the shared memory: a shallower ring measured
// faster than a deeper one (bf16 B x 2048 x 4096, us, two slots against
// the share's 3 at B16 / 8 at B8: minGRU 158.3 against 160.1 and 102.8
// against 105.1, decayed 184.7 against 184.6 and 115.4 against 119.2,
// MinMax 76.2 against 77.3 at B8), while half the blocks at a time with
// twice the share (a deeper ring, two waves) measured 193.0 at B16.
constexpr int kSeqPairMaxSlots = 2;
constexpr int kSeqWarpsPerBlock = 1;
constexpr size_t kAssumedSmemPerSM = 233472;
constexpr size_t kAssumedSmemReserved = 1024;
constexpr size_t kAssumedSmemPerBlock = 232448;

std::atomic<int> g_override_cg{0};
std::atomic<int> g_override_r{0};
std::atomic<int> g_override_kind{KIND_AUTO};
// Launch epochs tag the hand-off words (32 bits in each word).  0 never tags a
// word (zeroed memory) and 1 is reserved for launches captured into CUDA
// graphs, which zero the words inside the graph first.
std::atomic<uint64_t> g_epoch{2};
std::atomic<uint32_t> g_spin_limit{sgr::kSpinLimit};
std::atomic<int64_t> g_drop_tile{-1};

uint32_t next_epoch() {
    uint32_t e;
    do { e = uint32_t(g_epoch.fetch_add(1)); } while (e < 2);
    return e;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Plan {
    int esz = 4;          // bytes per stored element
    bool vec = false;     // 128-bit path
    int kind = KIND_TILE;
    int split = 1;        // channel-sequential: row groups per slot (1, or 2 half-warps)
    int V = 1;            // channels per thread
    int cg = 32;          // lanes across channels
    int r = 2;            // rows per thread
    int stages = 0;       // pipelined: tiles in flight per block
    int warps = kWarps;   // data warps per block
    int TR = 0, TC = 0;   // tile rows / channels
    int64_t n_dt = 0, n_chains = 0, n_chunks = 0, n_tiles = 0;
    size_t smem = 0;      // dynamic shared memory per block
    size_t off_words = 0, ws_bytes = 0;
};

bool mul_ok(int64_t a, int64_t b, int64_t *out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > std::numeric_limits<int64_t>::max() / a) return false;
    *out = a * b;
    return true;
}

// pipelined lane layout: fp32 8 lanes x 4 channels (32-channel tiles, 128-byte
// rows), bf16 16 lanes x 4 channels (64-channel tiles, 128-byte rows)
template <typename IO> constexpr int pipe_cg() { return sizeof(IO) == 4 ? 8 : 16; }

template <typename IO, int R, int W>
constexpr size_t pipe_smem() { return PipeShape<IO, 4, pipe_cg<IO>(), R, kStages, W>::smem_bytes; }

template <typename IO>
size_t pipe_smem_for(int r, bool wide) {
    if (r == 8) return wide ? pipe_smem<IO, 8, kPipeWarpsWide>() : pipe_smem<IO, 8, kPipeWarps>();
    if (wide) return r == 2 ? pipe_smem<IO, 2, kPipeWarpsWide>() : pipe_smem<IO, 4, kPipeWarpsWide>();
    return r == 2 ? pipe_smem<IO, 2, kPipeWarps>() : pipe_smem<IO, 4, kPipeWarps>();
}

// cuTensorMapEncodeTiled, fetched once from the driver through the runtime
// (no link-time dependency on the driver library)
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load();
    if (f == nullptr) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || ptr == nullptr)
            return nullptr;
        f = reinterpret_cast<EncodeTiledFn>(ptr);
        fn.store(f);
    }
    return f;
}

// Tensor map of one (B, T, D) operand for boxes of TC channels x TR rows x 1
// batch row; elements past the tensor's edges read as zero.
bool make_operand_map(CUtensorMap *map, const void *ptr, int64_t B, int64_t T, int64_t D, int esz,
                      int TC, int TR) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(T), cuuint64_t(B)};
    const cuuint64_t strides[2] = {cuuint64_t(D) * esz, cuuint64_t(T) * cuuint64_t(D) * esz};
    const cuuint32_t box[3] = {cuuint32_t(TC), cuuint32_t(TR), 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUtensorMapDataType dt = esz == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return enc(map, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shared memory of the channel-sequential kernel.  With K = ceil(groups /
// SMs) warps per SM in one wave, each single-warp block asks for about 1/K of
// the SM's shared memory, so no SM can take more than K of them and the
// groups spread evenly over the SMs (the block scheduler would otherwise be
// free to stack more on some SMs and leave others short); the share beyond
// the staging buffers deepens the load ring, up to kSeqMaxSlots slots.  Past
// 16 warps per SM the work runs in waves and the ring keeps 4 slots.
struct SeqLayout {
    int slots = 4;
    size_t smem = 0;
};
enum SeqKind { SEQ_SCAN = 0, SEQ_BACKWARD = 1, SEQ_FOLD = 2 };
size_t seq_bytes(int kind, int S, int row_bytes, size_t gap) {
    return kind == SEQ_BACKWARD ? seq_bwd_warp_bytes(S, row_bytes, gap)
         : kind == SEQ_FOLD     ? seq_fold_warp_bytes(S, row_bytes)
                                : seq_warp_bytes(S, row_bytes, gap);
}
// gap: per-slot bytes of time-decay gaps brought by the copy engine (0 or kSeqGapBytes)
SeqLayout seq_layout(int64_t groups, int row_bytes, int sms, size_t smem_sm, size_t reserved,
                     size_t smem_block_max, int backward = SEQ_SCAN, size_t gap = 0) {
    SeqLayout l;
    const int64_t K = sms > 0 ? (groups + sms - 1) / sms : 1;
    size_t alloc = seq_bytes(backward, 4, row_bytes, gap);
    if (K >= 1 && K <= 16) {
        const size_t share = smem_sm / size_t(K);
        alloc = share > reserved ? (share - reserved) / 128 * 128 : 0;
    }
    alloc = std::min(alloc, smem_block_max);
    int S = kSeqMaxSlots;
    while (S > kSeqMinSlots && seq_bytes(backward, S, row_bytes, gap) > alloc) --S;
    l.slots = S;
    l.smem = std::max(alloc, seq_bytes(backward, S, row_bytes, gap));
    return l;
}

// the two-warp blocks of scan_sequential_pair_kernel: one block per channel
// group asking for its share of the SM's shared memory (so that the groups
// spread evenly), of which its warps' rings take kSeqPairMaxSlots slots
// wide: the two-channels-per-lane form (64-channel groups, float4 exchange)
// with nw warps per group
SeqLayout seq_pair_layout(int64_t groups, int row_bytes, int sms, size_t smem_sm, size_t reserved,
                          size_t smem_block_max, size_t gap = 0, bool wide = false, int nw = kPairWarps) {
    auto bytes = [&](int S) {
        return wide ? seq_pair2_block_bytes(S, gap, nw) : seq_pair_block_bytes(S, row_bytes, gap);
    };
    SeqLayout l;
    const int64_t K = sms > 0 ? (groups + sms - 1) / sms : 1;
    size_t alloc = bytes(4);
    if (K >= 1 && K <= 16) {
        const size_t share = smem_sm / size_t(K);
        alloc = share > reserved ? (share - reserved) / 128 * 128 : 0;
    }
    alloc = std::min(alloc, smem_block_max);
    int S = kSeqPairMaxSlots;
    while (S > kSeqMinSlots && bytes(S) > alloc) --S;
    l.slots = S;
    l.smem = std::max(alloc, bytes(S));
    return l;
}

// Tile shape of a scan.  Aligned vector-width rows take the pipelined kernel
// (fp32: 7 x 4 x R rows x 32 channels; bf16: 7 x 2 x R rows x 64 channels;
// 128-byte row segments); anything else takes the tile kernel's scalar
// variant.  The override knobs select the kernel and the rows per thread.
// force_tile: the tile kernel whatever the alignment (the gradient kernel,
// which keeps four values per element live, also caps a thread at 16 elements).
// light_op: the recurrence does next to no arithmetic per element (MinMax), so
// per-tile work dominates and the longer tiles of 15-warp blocks pay wherever
// they still give every SM 4 tiles (measured: MinMax B4 x 8192 x 768 fp32 0.81
// of the copy bandwidth against 0.78 with 7-warp blocks; minGRU slower).
// decay: the time-decayed minGRU, which takes the plain scan's plans (bf16:
// 8 rows per thread in 7-warp blocks, measured 78.3 against 82.4 us with 4
// rows in 15-warp blocks on B8 x 4096 x 1024, 41.5 against 45.5 us on B2 x
// 2048 x 4096, 47.5 against 47.7 us on B4 x 8192 x 512); wide decayed
// batches take the channel-sequential kernels like the plain scan, bf16 ones
// from kSeqQuadFrom groups per SM with four warps per 64-channel group
// (each slot's gaps arrive with it through the copy engine, or, for gap
// arrays the copy engine cannot address, spread across the lanes two slots
// ahead)
// chunked_only: never the channel-sequential kernels (the log-space minGRU,
// which only the chunked kernels evaluate)
Plan make_plan(int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype, bool aligned,
               bool force_tile = false, bool light_op = false, bool decay = false,
               bool chunked_only = false) {
    Plan p;
    p.esz = (dtype == SGR_BF16) ? 2 : 4;
    const int vw = 16 / p.esz;
    p.vec = aligned && (D % vw == 0);
    const int ok = g_override_kind.load();
    {
        // whole sequences per warp when the channel groups fill the GPU
        const int64_t cw = 32;
        const int64_t groups = B * ((D + cw - 1) / cw);
        const bool seq_ok = p.vec && !force_tile && !chunked_only && T <= int64_t(std::numeric_limits<int>::max()) &&
                            B <= int64_t(std::numeric_limits<int>::max());
        const int min_per_sm = p.esz == 2 ? kSeqMinWarpsPerSMHalf : kSeqMinWarpsPerSM;
        const bool want = seq_kind(ok) || (ok == KIND_AUTO && groups >= int64_t(min_per_sm) * kAssumedSMs);
        if (seq_ok && want) {
            const bool split = ok == KIND_SEQUENTIAL_SPLIT;
            const int pair_below = p.esz == 2 ? kSeqPairBelowHalf : kSeqPairBelow;
            // two channels per lane: bf16 only; automatic from kSeqPairBelowHalf
            // groups per SM, where it keeps the one-warp kernel's warp count
            // with fewer instructions and 128-byte rows
            // four warps per group of 64 channels (8 rows of each slot per warp)
            const bool auto_quad = p.esz == 2 && ok == KIND_AUTO &&
                                   (light_op || (groups >= int64_t(kSeqQuadFrom) * kAssumedSMs &&
                                                 (decay || groups < int64_t(pair_below) * kAssumedSMs)));
            const bool wide = p.esz == 2 && (ok == KIND_SEQUENTIAL_PAIR2 || ok == KIND_SEQUENTIAL_QUAD || auto_quad ||
                                             (ok == KIND_AUTO && groups >= int64_t(pair_below) * kAssumedSMs));
            const bool quad = wide && (ok == KIND_SEQUENTIAL_QUAD || auto_quad);
            const int nw = quad ? kQuadWarps : kPairWarps;
            const bool pair = wide || ok == KIND_SEQUENTIAL_PAIR || ok == KIND_SEQUENTIAL_PAIR2 ||
                              ok == KIND_SEQUENTIAL_QUAD ||
                              (ok == KIND_AUTO && groups < int64_t(pair_below) * kAssumedSMs);
            const int64_t gw = wide ? int64_t(kPair2Channels) : split ? cw / 2 : cw;   // channels per warp
            const int64_t n_warps = B * ((D + gw - 1) / gw);
            const size_t gap = decay ? kSeqGapBytes : 0;
            const SeqLayout lay = pair ? seq_pair_layout(n_warps, int(gw) * p.esz, kAssumedSMs, kAssumedSmemPerSM,
                                                         kAssumedSmemReserved, kAssumedSmemPerBlock, gap, wide, nw)
                                       : seq_layout(n_warps, int(gw) * p.esz, kAssumedSMs, kAssumedSmemPerSM,
                                                    kAssumedSmemReserved, kAssumedSmemPerBlock, SEQ_SCAN, gap);
            p.kind = quad ? KIND_SEQUENTIAL_QUAD : wide ? KIND_SEQUENTIAL_PAIR2 : pair ? KIND_SEQUENTIAL_PAIR
                                                      : split ? KIND_SEQUENTIAL_SPLIT : KIND_SEQUENTIAL;
            p.split = (split || pair) ? 2 : 1;
            p.V = wide ? 2 : 1;
            p.cg = int(gw / p.V);                                  // lanes across a group's channels
            p.r = pair ? 32 / nw : kSeqRows / p.split;             // rows of a slot per lane
            p.stages = lay.slots;
            p.warps = pair ? nw : kSeqWarpsPerBlock;
            p.TR = T > 0 ? int(std::min<int64_t>(T, std::numeric_limits<int>::max())) : 0;
            p.TC = int(gw);
            p.smem = lay.smem;
            p.n_dt = (D + gw - 1) / gw;
            p.n_chains = B * p.n_dt;
            p.n_chunks = T > 0 ? 1 : 0;
            p.n_tiles = p.n_chains * p.n_chunks;
            if (p.n_tiles > 0) {
                p.off_words = kAlign;                           // the header alone: status word
                p.ws_bytes = kAlign;
            }
            return p;
        }
    }
    p.kind = (p.vec && ok != KIND_TILE && !force_tile) ? KIND_PIPELINED : KIND_TILE;
    if (p.kind == KIND_PIPELINED && ok == KIND_AUTO) {
        // under two tiles per persistent block: little to pipeline, and
        // one plain launch per tile starts sooner (no tensor maps, no
        // cooperative launch)
        const int64_t tc = p.esz == 4 ? 32 : 64, tr = 112;
        const int64_t tiles = B * ((D + tc - 1) / tc) * ((T + tr - 1) / tr);
        if (tiles < 4 * kAssumedSMs) p.kind = KIND_TILE;
    }
    const int orr = g_override_r.load();
    if (p.kind == KIND_PIPELINED) {
        // 4 channels per lane (16-byte fp32 / 8-byte bf16 vectors)
        p.V = 4;
        p.cg = p.esz == 4 ? 8 : 16;
        p.TC = p.cg * p.V;
        // rows per thread {2, 4, 8}; automatic: 4 for fp32, 8 for bf16, whose
        // elements are half the bytes, so per-tile work (warp scan, barriers,
        // hand-off) weighs twice as much per byte and is spread over twice
        // the rows (replayed without the one-tile lag, see the kernel)
        p.r = (orr == 2 || orr == 4 || orr == 8) ? orr : (p.esz == 2 ? 8 : 4);
        p.stages = kStages;
        // Block shape: about (blocks in flight) / n_chains chunks of one
        // channel tile are processed at once and a look-back folds that many
        // summaries; when that depth reaches 8 with two 8-warp blocks per SM,
        // one 16-warp block per SM with tiles twice as long halves it.
        // Only when the wide tiles still give every SM at least 4 of them.
        const int64_t n_chains = B * ((D + p.TC - 1) / p.TC);
        const int64_t tr_wide = int64_t(kPipeWarpsWide) * (32 / p.cg) * p.r;
        const int64_t tiles_wide = n_chains * ((T + tr_wide - 1) / tr_wide);
        bool wide = n_chains > 0 && (light_op || 2 * kAssumedSMs >= 8 * n_chains) &&
                    tiles_wide >= 4 * kAssumedSMs;
        if (ok == KIND_PIPELINED) wide = false;
        if (ok == KIND_PIPELINED_WIDE) wide = true;
        // 8 rows: bf16 only (fp32 tiles of 8 rows exceed the TMA box with 15
        // warps and leave shared memory for one 7-warp block per SM)
        if (p.r == 8 && p.esz == 4) p.r = 4;
        p.kind = wide ? KIND_PIPELINED_WIDE : KIND_PIPELINED;
        p.warps = wide ? kPipeWarpsWide : kPipeWarps;
        p.TR = p.warps * (32 / p.cg) * p.r;
        p.smem = p.esz == 4 ? pipe_smem_for<float>(p.r, wide) : pipe_smem_for<__nv_bfloat16>(p.r, wide);
    } else {
        // tile kernel: 8 lanes x one vector (32 fp32 / 64 bf16 channels,
        // 128-byte row segments) or, unaligned, 32 lanes x 1 channel
        p.V = p.vec ? vw : 1;
        p.cg = p.vec ? 8 : 32;
        p.TC = p.cg * p.V;
        const int J = 32 / p.cg;
        const int64_t n_chains = B * ((D + p.TC - 1) / p.TC);
        // rows per thread: the automatic choice keeps a data thread within 72
        // registers (16 elements of each operand); the override may go to 32
        const int rmax_auto = p.vec ? (p.V >= 8 ? 2 : 4) : 8;
        const int rmax = p.V >= 8 ? 4 : 8;
        int r = 1;
        if (orr == 1 || orr == 2 || orr == 4 || orr == 8) {
            r = orr < rmax ? orr : rmax;
        } else {
            for (int cand : {8, 4, 2, 1}) {
                if (cand > rmax_auto) continue;
                const int64_t tr = int64_t(kWarps) * J * cand;
                const int64_t chunks = (T + tr - 1) / tr;
                if (n_chains * chunks >= kTargetTiles || cand == 1) { r = cand; break; }
            }
        }
        if (force_tile) {
            while (r > 1 && r * p.V > 16) r /= 2;
        }
        p.r = r;
        p.TR = kWarps * J * r;
    }
    p.n_dt = (D + p.TC - 1) / p.TC;
    p.n_chains = B * p.n_dt;
    p.n_chunks = (T + p.TR - 1) / p.TR;
    p.n_tiles = p.n_chains * p.n_chunks;
    if (p.n_tiles > 0) {
        p.off_words = kAlign;                                   // [0, 256): header
        p.ws_bytes = kAlign;
        if (p.n_chunks > 1) p.ws_bytes = align_up(p.off_words + size_t(p.n_tiles) * 3 * p.TC * 8, kAlign);
    }
    return p;
}

// divisor constants for FastDiv (see scan_engine.cuh); 1 <= d < 2^31
FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    uint32_t s = 0;
    while ((uint64_t(1) << s) < d) ++s;
    f.s = s;
    f.m = uint32_t(((uint64_t(1) << 32) * ((uint64_t(1) << s) - d)) / d + 1);
    return f;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// bytes spanned by B rows of D elements with a batch stride (stride 0 = one row)
size_t rows_span(int64_t B, int64_t D, int64_t bs, int esz) {
    if (B <= 0 || D <= 0) return 0;
    return size_t((B - 1) * bs + D) * esz;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
    int sms = 0;
};
DeviceInfo device_info(int dev) {
    static std::atomic<int> cache[64];
    DeviceInfo d;
    if (dev >= 0 && dev < 64) {
        int v = cache[dev].load();
        if (v == 0) {
            if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) v = 0;
            cache[dev].store(v);
        }
        d.sms = v;
    }
    return d;
}

// ---- tile kernel launch
// Blocks of a tile-kernel launch: one per tile without a ticket counter;
// with one, as many as stay resident at once (the blocks loop over tickets),
// from the kernel's occupancy on the current device, read once per kernel
// and device.
template <class Kernel>
cudaError_t tile_grid(Kernel kernel, int threads, int64_t n_tiles, bool ticket, int64_t *grid) {
    *grid = n_tiles;
    if (!ticket) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    static std::mutex mu;
    static std::vector<std::pair<std::pair<const void *, int>, int>> cache;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(reinterpret_cast<const void *>(kernel), dev);
    int per_sm = 0;
    for (const auto &c : cache)
        if (c.first == key) per_sm = c.second;
    if (per_sm == 0) {
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0)) != cudaSuccess) return e;
        if (per_sm <= 0) return cudaErrorInvalidConfiguration;
        cache.emplace_back(key, per_sm);
    }
    const DeviceInfo di = device_info(dev);
    if (di.sms <= 0) return cudaErrorInvalidDevice;
    *grid = std::min<int64_t>(n_tiles, int64_t(per_sm) * di.sms);
    return cudaSuccess;
}

template <class Op, typename IO, int V, int CG, int R>
cudaError_t launch_tile(const ScanParams &sp, cudaStream_t s) {
    if constexpr (R * V > 32) {
        return cudaErrorInvalidConfiguration;   // never planned (see make_plan)
    } else {
        // registers a data thread keeps live: its tile (2RV), one pair per
        // channel (2V) and about 24 for addressing; blocks of 256 threads
        constexpr int NEED = 2 * R * V + 2 * V + 24;
        constexpr int MINB = NEED <= 56 ? 4 : (NEED <= 72 ? 3 : 2);
        auto kernel = scan_tile_kernel<Op, IO, V, CG, R, kWarps, MINB>;
        int64_t grid = 0;
        const cudaError_t e = tile_grid(kernel, (kWarps + 1) * 32, sp.n_tiles, sp.ticket != nullptr, &grid);
        if (e != cudaSuccess) return e;
        kernel<<<dim3(unsigned(grid)), (kWarps + 1) * 32, 0, s>>>(sp);
        return cudaGetLastError();
    }
}

template <class Op, typename IO, int V, int CG>
cudaError_t dispatch_tile_r(const Plan &pl, const ScanParams &sp, cudaStream_t s) {
    switch (pl.r) {
        case 1: return launch_tile<Op, IO, V, CG, 1>(sp, s);
        case 2: return launch_tile<Op, IO, V, CG, 2>(sp, s);
        case 4: return launch_tile<Op, IO, V, CG, 4>(sp, s);
        default: return launch_tile<Op, IO, V, CG, 8>(sp, s);
    }
}

// ---- pipelined kernel launch: persistent, co-resident blocks

// Tensor maps of a decay's gaps (B, T) fp32 rows with a batch stride and
// rates (D,) fp32, for boxes of TR gaps of one batch row and TC rates; false
// when the copy engine cannot take them (16-byte aligned bases and row
// stride needed), and the kernel then loads them itself.
bool make_decay_maps(CUtensorMap *gap, CUtensorMap *lam, const ScanParams &sp, int TR, int TC) {
    if (!sp.decay_dt || !sp.decay_lam || !aligned16(sp.decay_dt) || !aligned16(sp.decay_lam)) return false;
    if (sp.B > 1 && (sp.decay_dt_bs % 4) != 0) return false;
    EncodeTiledFn enc = encode_tiled_fn();
    if (enc == nullptr) return false;
    {
        const cuuint64_t dims[2] = {cuuint64_t(sp.T), cuuint64_t(sp.B)};
        const cuuint64_t row = sp.B > 1 ? cuuint64_t(sp.decay_dt_bs) * 4 : (cuuint64_t(sp.T) * 4 + 15) / 16 * 16;
        const cuuint64_t strides[1] = {row};
        const cuuint32_t box[2] = {cuuint32_t(TR), 1u};
        const cuuint32_t es[2] = {1u, 1u};
        if (enc(gap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(sp.decay_dt), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    {
        const cuuint64_t dims[1] = {cuuint64_t(sp.D)};
        const cuuint64_t strides[1] = {0};
        const cuuint32_t box[1] = {cuuint32_t(TC)};
        const cuuint32_t es[1] = {1u};
        if (enc(lam, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, const_cast<float *>(sp.decay_lam), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    return true;
}

// Tensor map of a decay's gaps for the channel-sequential kernels: boxes of
// 16 gaps of one batch row (64 bytes); false when the copy engine cannot take
// the array (16-byte aligned base and row stride needed), and the kernels
// then load the gaps themselves.
bool make_seq_gap_map(CUtensorMap *gap, const ScanParams &sp) {
    if (!sp.decay_dt || !aligned16(sp.decay_dt)) return false;
    if (sp.B > 1 && (sp.decay_dt_bs % 4) != 0) return false;
    EncodeTiledFn enc = encode_tiled_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {cuuint64_t(sp.T), cuuint64_t(sp.B)};
    const cuuint64_t row = sp.B > 1 ? cuuint64_t(sp.decay_dt_bs) * 4 : (cuuint64_t(sp.T) * 4 + 15) / 16 * 16;
    const cuuint64_t strides[1] = {row};
    const cuuint32_t box[2] = {cuuint32_t(kSeqRows), 1u};
    const cuuint32_t es[2] = {1u, 1u};
    return enc(gap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(sp.decay_dt), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class Op, typename IO, int V, int R, int W, bool DT>
cudaError_t launch_pipelined_shape(const ScanParams &sp_in, const CUtensorMap &map0, const CUtensorMap &map1,
                                   const CUtensorMap &map_gap, const CUtensorMap &map_lam, cudaStream_t s,
                                   int64_t *grid_out) {
    constexpr int CG = pipe_cg<IO>();
    using Shape = PipeShape<IO, V, CG, R, kStages, W, DT>;
    constexpr int MINB = W == kPipeWarps ? 2 : 1;
    auto kernel = scan_pipelined_kernel<Op, IO, V, CG, R, kStages, W, MINB, DT>;
    constexpr size_t smem = Shape::smem_bytes;
    constexpr int NT = (W + 1) * 32;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    // per-device one-time set-up of the shared-memory limit and occupancy
    static std::atomic<int> occ_cache[64];
    int occ = (dev >= 0 && dev < 64) ? occ_cache[dev].load() : 0;
    if (occ == 0) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, NT, smem);
        if (e != cudaSuccess) return e;
        if (occ <= 0) return cudaErrorInvalidConfiguration;
        if (dev >= 0 && dev < 64) occ_cache[dev].store(occ);
    }
    const DeviceInfo di = device_info(dev);
    if (di.sms <= 0) return cudaErrorInvalidDevice;
    const int64_t grid = std::min<int64_t>(sp_in.n_tiles, int64_t(di.sms) * occ);
    if (grid_out) *grid_out = grid;
    ScanParams sp = sp_in;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, sp, map0, map1, map_gap, map_lam);
}

template <class Op, typename IO, int V, int R, int W>
cudaError_t launch_pipelined(const ScanParams &sp_in, cudaStream_t s, int64_t *grid_out) {
    constexpr int CG = pipe_cg<IO>();
    using Shape = PipeShape<IO, V, CG, R, kStages, W>;
    alignas(64) CUtensorMap map0, map1, map_gap, map_lam;
    if (!make_operand_map(&map0, sp_in.in0, sp_in.B, sp_in.T, sp_in.D, int(sizeof(IO)), Shape::TC, Shape::TR) ||
        !make_operand_map(&map1, sp_in.in1, sp_in.B, sp_in.T, sp_in.D, int(sizeof(IO)), Shape::TC, Shape::TR))
        return cudaErrorInvalidValue;
    if constexpr (Op::kDecay && PipeShape<IO, V, CG, R, kStages, W, true>::dec_boxable) {
        if (make_decay_maps(&map_gap, &map_lam, sp_in, Shape::TR, Shape::TC))
            return launch_pipelined_shape<Op, IO, V, R, W, true>(sp_in, map0, map1, map_gap, map_lam, s, grid_out);
    }
    // no decay operands through the copy engine: the two maps are not read
    return launch_pipelined_shape<Op, IO, V, R, W, false>(sp_in, map0, map1, map0, map1, s, grid_out);
}

// ---- channel-sequential kernels: one warp per channel group
// Per device: SM count and shared-memory figures, read once; and, once per
// kernel and device, the kernel's dynamic shared-memory limit raised to the
// device's maximum per block.
struct SeqDev {
    int sms = 0, smem_sm = 0, reserved = 0, smem_block = 0;
};
cudaError_t seq_device(const void *kernel, size_t min_bytes, SeqDev *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    static std::mutex mu;
    static SeqDev info[64];
    static bool have[64];
    static std::vector<std::pair<const void *, int>> raised;
    std::lock_guard<std::mutex> lock(mu);
    if (!have[dev]) {
        SeqDev d;
        if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&d.smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) !=
            cudaSuccess)
            return e;
        if ((e = cudaDeviceGetAttribute(&d.reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess)
            return e;
        if ((e = cudaDeviceGetAttribute(&d.smem_block, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
            cudaSuccess)
            return e;
        if (d.sms <= 0) return cudaErrorInvalidConfiguration;
        info[dev] = d;
        have[dev] = true;
    }
    if (size_t(info[dev].smem_block) < min_bytes) return cudaErrorInvalidConfiguration;
    if (std::find(raised.begin(), raised.end(), std::make_pair(kernel, dev)) == raised.end()) {
        if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, info[dev].smem_block)) !=
            cudaSuccess)
            return e;
        raised.emplace_back(kernel, dev);
    }
    *out = info[dev];
    return cudaSuccess;
}
template <class Op, typename IO, int SPLIT, bool DT>
cudaError_t launch_sequential_dt(const Plan &pl, const ScanParams &sp, const CUtensorMap &map0,
                                 const CUtensorMap &map1, const CUtensorMap &map_out, const CUtensorMap &map_gap,
                                 cudaStream_t s) {
    constexpr int WB = kSeqWarpsPerBlock;
    constexpr int CW = 32 / SPLIT;
    constexpr int kRowBytes = CW * int(sizeof(IO));
    constexpr size_t kGap = DT ? kSeqGapBytes : 0;
    auto kernel = scan_sequential_kernel<Op, IO, WB, SPLIT, DT>;
    SeqDev d;
    cudaError_t e = seq_device(reinterpret_cast<const void *>(kernel), seq_warp_bytes(kSeqMinSlots, kRowBytes, kGap), &d);
    if (e != cudaSuccess) return e;
    SeqParams q;
    q.s = sp;
    q.n_groups = pl.n_dt;
    q.n_warps = pl.n_chains;
    const SeqLayout lay = seq_layout((q.n_warps + WB - 1) / WB * WB, kRowBytes, d.sms, size_t(d.smem_sm),
                                     size_t(d.reserved), size_t(d.smem_block), SEQ_SCAN, kGap);
    q.slots = lay.slots;
    const int64_t grid = (q.n_warps + WB - 1) / WB;
    kernel<<<dim3(unsigned(grid)), WB * 32, lay.smem, s>>>(q, map0, map1, map_out, map_gap);
    return cudaGetLastError();
}

template <class Op, typename IO, int SPLIT>
cudaError_t launch_sequential(const Plan &pl, const ScanParams &sp, cudaStream_t s) {
    constexpr int CW = 32 / SPLIT;
    alignas(64) CUtensorMap map0, map1, map_out, map_gap;
    if (!make_operand_map(&map0, sp.in0, sp.B, sp.T, sp.D, int(sizeof(IO)), CW, kSeqRows) ||
        !make_operand_map(&map1, sp.in1, sp.B, sp.T, sp.D, int(sizeof(IO)), CW, kSeqRows) ||
        !make_operand_map(&map_out, sp.out, sp.B, sp.T, sp.D, int(sizeof(IO)), CW, kSeqRows))
        return cudaErrorInvalidValue;
    if constexpr (Op::kDecay) {
        if (make_seq_gap_map(&map_gap, sp))
            return launch_sequential_dt<Op, IO, SPLIT, true>(pl, sp, map0, map1, map_out, map_gap, s);
    }
    // no gaps through the copy engine: the kernel does not read map_gap
    return launch_sequential_dt<Op, IO, SPLIT, false>(pl, sp, map0, map1, map_out, map0, s);
}

template <class Op, typename IO, bool DT>
cudaError_t launch_sequential_pair_dt(const Plan &pl, const ScanParams &sp, const CUtensorMap &map0,
                                      const CUtensorMap &map1, const CUtensorMap &map_out,
                                      const CUtensorMap &map_gap, cudaStream_t s) {
    constexpr int kRowBytes = 32 * int(sizeof(IO));
    constexpr size_t kGap = DT ? kSeqGapBytes : 0;
    auto kernel = scan_sequential_pair_kernel<Op, IO, DT>;
    SeqDev d;
    cudaError_t e = seq_device(reinterpret_cast<const void *>(kernel),
                               seq_pair_block_bytes(kSeqMinSlots, kRowBytes, kGap), &d);
    if (e != cudaSuccess) return e;
    SeqParams q;
    q.s = sp;
    q.n_groups = pl.n_dt;
    q.n_warps = pl.n_chains;                  // channel groups: one block each
    const SeqLayout lay = seq_pair_layout(q.n_warps, kRowBytes, d.sms, size_t(d.smem_sm), size_t(d.reserved),
                                          size_t(d.smem_block), kGap);
    q.slots = lay.slots;
    kernel<<<dim3(unsigned(q.n_warps)), kPairWarps * 32, lay.smem, s>>>(q, map0, map1, map_out, map_gap);
    return cudaGetLastError();
}

template <class Op, typename IO>
cudaError_t launch_sequential_pair(const Plan &pl, const ScanParams &sp, cudaStream_t s) {
    constexpr int CW = 32;
    alignas(64) CUtensorMap map0, map1, map_out, map_gap;
    if (!make_operand_map(&map0, sp.in0, sp.B, sp.T, sp.D, int(sizeof(IO)), CW, kSeqRows) ||
        !make_operand_map(&map1, sp.in1, sp.B, sp.T, sp.D, int(sizeof(IO)), CW, kSeqRows) ||
        !make_operand_map(&map_out, sp.out, sp.B, sp.T, sp.D, int(sizeof(IO)), CW, kSeqRows))
        return cudaErrorInvalidValue;
    if constexpr (Op::kDecay) {
        if (make_seq_gap_map(&map_gap, sp))
            return launch_sequential_pair_dt<Op, IO, true>(pl, sp, map0, map1, map_out, map_gap, s);
    }
    return launch_sequential_pair_dt<Op, IO, false>(pl, sp, map0, map1, map_out, map0, s);
}

template <class Op, bool DT, int NW>
cudaError_t launch_sequential_pair2_dt(const Plan &pl, const ScanParams &sp, const CUtensorMap &map0,
                                       const CUtensorMap &map1, const CUtensorMap &map_out,
                                       const CUtensorMap &map_gap, cudaStream_t s) {
    constexpr size_t kGap = DT ? kSeqGapBytes : 0;
    auto kernel = scan_sequential_pair2_kernel<Op, DT, NW>;
    SeqDev d;
    cudaError_t e =
        seq_device(reinterpret_cast<const void *>(kernel), seq_pair2_block_bytes(kSeqMinSlots, kGap, NW), &d);
    if (e != cudaSuccess) return e;
    SeqParams q;
    q.s = sp;
    q.n_groups = pl.n_dt;
    q.n_warps = pl.n_chains;                  // channel groups: one block each
    const SeqLayout lay = seq_pair_layout(q.n_warps, kPair2Channels * 2, d.sms, size_t(d.smem_sm), size_t(d.reserved),
                                          size_t(d.smem_block), kGap, true, NW);
    q.slots = lay.slots;
    kernel<<<dim3(unsigned(q.n_warps)), NW * 32, lay.smem, s>>>(q, map0, map1, map_out, map_gap);
    return cudaGetLastError();
}

// NW warps per group of 64 channels, each taking 32 / NW rows of a slot (the
// height of the operand and output boxes)
template <class Op, int NW>
cudaError_t launch_sequential_pair2(const Plan &pl, const ScanParams &sp, cudaStream_t s) {
    constexpr int CW = kPair2Channels;
    constexpr int RW = 32 / NW;
    alignas(64) CUtensorMap map0, map1, map_out, map_gap;
    if (!make_operand_map(&map0, sp.in0, sp.B, sp.T, sp.D, 2, CW, RW) ||
        !make_operand_map(&map1, sp.in1, sp.B, sp.T, sp.D, 2, CW, RW) ||
        !make_operand_map(&map_out, sp.out, sp.B, sp.T, sp.D, 2, CW, RW))
        return cudaErrorInvalidValue;
    if constexpr (Op::kDecay) {
        if (make_seq_gap_map(&map_gap, sp))
            return launch_sequential_pair2_dt<Op, true, NW>(pl, sp, map0, map1, map_out, map_gap, s);
    }
    return launch_sequential_pair2_dt<Op, false, NW>(pl, sp, map0, map1, map_out, map0, s);
}

template <class Op, typename IO>
cudaError_t dispatch(const Plan &pl, const ScanParams &sp, cudaStream_t s) {
    constexpr int VW = 16 / int(sizeof(IO));
    if constexpr (!Op::kLogSpace) {
        if (pl.kind == KIND_SEQUENTIAL) return launch_sequential<Op, IO, 1>(pl, sp, s);
        if (pl.kind == KIND_SEQUENTIAL_SPLIT) return launch_sequential<Op, IO, 2>(pl, sp, s);
        if (pl.kind == KIND_SEQUENTIAL_PAIR) return launch_sequential_pair<Op, IO>(pl, sp, s);
        if (pl.kind == KIND_SEQUENTIAL_PAIR2 || pl.kind == KIND_SEQUENTIAL_QUAD) {
            if constexpr (sizeof(IO) == 2) {
                if (pl.kind == KIND_SEQUENTIAL_QUAD) return launch_sequential_pair2<Op, kQuadWarps>(pl, sp, s);
                return launch_sequential_pair2<Op, kPairWarps>(pl, sp, s);
            } else {
                return cudaErrorInvalidConfiguration;    // never planned (bf16 only)
            }
        }
    } else {
        if (seq_kind(pl.kind)) return cudaErrorInvalidConfiguration;    // never planned (chunked_only)
    }
    if (pl.kind == KIND_PIPELINED) {
        if constexpr (sizeof(IO) == 2) {
            if (pl.r == 8) return launch_pipelined<Op, IO, 4, 8, kPipeWarps>(sp, s, nullptr);
        }
        return pl.r == 2 ? launch_pipelined<Op, IO, 4, 2, kPipeWarps>(sp, s, nullptr)
                         : launch_pipelined<Op, IO, 4, 4, kPipeWarps>(sp, s, nullptr);
    }
    if (pl.kind == KIND_PIPELINED_WIDE) {
        if constexpr (sizeof(IO) == 2) {
            if (pl.r == 8) return launch_pipelined<Op, IO, 4, 8, kPipeWarpsWide>(sp, s, nullptr);
        }
        return pl.r == 2 ? launch_pipelined<Op, IO, 4, 2, kPipeWarpsWide>(sp, s, nullptr)
                         : launch_pipelined<Op, IO, 4, 4, kPipeWarpsWide>(sp, s, nullptr);
    }
    if (!pl.vec) return dispatch_tile_r<Op, IO, 1, 32>(pl, sp, s);
    return dispatch_tile_r<Op, IO, VW, 8>(pl, sp, s);
}

// time-decay arguments of the minGRU scans (null: no decay)
struct DecayArgs {
    const float *dt = nullptr;
    int64_t dt_bs = 0;
    const float *lam = nullptr;
    int log1p = 0;
};

sgr_status_t check_decay(const DecayArgs *dec, int64_t B, int64_t T, int64_t D) {
    if (!dec) return SGR_OK;
    if (!dec->dt || !dec->lam || dec->dt_bs < 0) return SGR_ERR_INVALID_ARG;
    if (B > 1 && dec->dt_bs < T) return SGR_ERR_INVALID_ARG;   // rows of gaps would overlap
    int64_t tmp = 0;
    if (!mul_ok(B - 1, dec->dt_bs, &tmp) || !mul_ok(tmp + T, 4, &tmp)) return SGR_ERR_UNSUPPORTED;
    (void)D;
    return SGR_OK;
}

// bytes the gaps span (B rows of T, batch stride dt_bs; sizes checked by
// check_decay) and the rates span
size_t decay_gap_bytes(const DecayArgs &dec, int64_t B, int64_t T) {
    return size_t((B - 1) * dec.dt_bs + T) * sizeof(float);
}
size_t decay_lam_bytes(int64_t D) { return size_t(D) * sizeof(float); }

// an output written while the gaps and rates are still being read must not
// share memory with them
bool overlaps_decay(const DecayArgs *dec, const void *out, size_t n, int64_t B, int64_t T, int64_t D) {
    return dec && (overlaps(out, n, dec->dt, decay_gap_bytes(*dec, B, T)) ||
                   overlaps(out, n, dec->lam, decay_lam_bytes(D)));
}

void set_decay(ScanParams &sp, const DecayArgs *dec) {
    if (!dec) return;
    sp.decay_dt = dec->dt;
    sp.decay_dt_bs = dec->dt_bs;
    sp.decay_lam = dec->lam;
    sp.decay_log1p = dec->log1p ? 1 : 0;
}

sgr_status_t run_scan(sgr_op_t op, const void *in0, const void *in1, const void *init,
                      int64_t init_bs, void *out, int64_t B, int64_t T, int64_t D,
                      sgr_dtype_t dtype, void *ws, size_t ws_bytes, cudaStream_t stream,
                      const DecayArgs *dec = nullptr) {
    if (dtype != SGR_F32 && dtype != SGR_BF16) return SGR_ERR_INVALID_ARG;
    if (op != SGR_OP_MINGRU && op != SGR_OP_MINMAX && op != SGR_OP_MINGRU_LOG) return SGR_ERR_INVALID_ARG;
    if (op == SGR_OP_MINGRU_LOG && dec) return SGR_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || D < 0 || init_bs < 0) return SGR_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || D == 0) return SGR_OK;
    if (!in0 || !in1 || !out) return SGR_ERR_INVALID_ARG;
    const sgr_status_t dst = check_decay(dec, B, T, D);
    if (dst != SGR_OK) return dst;
    const int esz = dtype == SGR_BF16 ? 2 : 4;
    int64_t n = 0, nbytes = 0;
    if (!mul_ok(B, T, &n) || !mul_ok(n, D, &n) || !mul_ok(n, esz, &nbytes)) return SGR_ERR_UNSUPPORTED;
    int64_t init_span_elems = 0;
    if (init && !mul_ok(B - 1, init_bs, &init_span_elems)) return SGR_ERR_UNSUPPORTED;
    const size_t tb = size_t(nbytes);
    const size_t ib = init ? rows_span(B, D, init_bs, esz) : 0;
    if (overlaps(out, tb, in0, tb) || overlaps(out, tb, in1, tb) || overlaps(out, tb, init, ib) ||
        overlaps_decay(dec, out, tb, B, T, D))
        return SGR_ERR_INVALID_ARG;

    const bool aligned = aligned16(in0) && aligned16(in1) && aligned16(out);
    const Plan pl = make_plan(B, T, D, dtype, aligned, false, op == SGR_OP_MINMAX, dec != nullptr,
                              op == SGR_OP_MINGRU_LOG);
    if (pl.n_tiles > int64_t(std::numeric_limits<int>::max())) return SGR_ERR_UNSUPPORTED;

    ScanParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.in0 = in0; sp.in1 = in1; sp.init = init; sp.init_bs = init_bs; sp.out = out;
    sp.B = B; sp.T = T; sp.D = D;
    sp.n_dt = pl.n_dt; sp.n_chains = pl.n_chains; sp.n_chunks = pl.n_chunks; sp.n_tiles = pl.n_tiles;
    sp.by_chains = make_fastdiv(uint32_t(pl.n_chains));
    sp.by_dt = make_fastdiv(uint32_t(pl.n_dt));
    sp.epoch = 0;
    sp.spin_limit = g_spin_limit.load();
    sp.drop_tile = g_drop_tile.load();
    set_decay(sp, dec);
    // every plan records its bounded waits in the workspace's status word
    if (!ws || ws_bytes < pl.ws_bytes || !aligned16(ws)) return SGR_ERR_WORKSPACE;
    sp.status = static_cast<uint32_t *>(ws);
    if (pl.n_chunks > 1) {
        char *w = static_cast<char *>(ws);
        sp.words = reinterpret_cast<uint64_t *>(w + pl.off_words);
        if (pl.kind == KIND_TILE) {
            // one block per tile: tiles go out by ticket in block start order
            sp.ticket = reinterpret_cast<uint32_t *>(w + kTicketOffset);
            if (cudaMemsetAsync(sp.ticket, 0, sizeof(uint32_t), stream) != cudaSuccess) return SGR_ERR_CUDA;
        }
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return SGR_ERR_CUDA;
        if (cs == cudaStreamCaptureStatusActive) {
            // a graph replays its launch arguments: clear the words inside the
            // graph so the fixed epoch of captured launches never sees stale ones
            if (cudaMemsetAsync(sp.words, 0, pl.ws_bytes - pl.off_words, stream) != cudaSuccess)
                return SGR_ERR_CUDA;
            sp.epoch = 1;
        } else {
            sp.epoch = next_epoch();
        }
    }
    cudaError_t e;
    if (op == SGR_OP_MINGRU && dec) {
        e = dtype == SGR_F32 ? dispatch<MinGRUDecayOp, float>(pl, sp, stream)
                             : dispatch<MinGRUDecayOp, __nv_bfloat16>(pl, sp, stream);
    } else if (op == SGR_OP_MINGRU) {
        e = dtype == SGR_F32 ? dispatch<MinGRUOp, float>(pl, sp, stream)
                             : dispatch<MinGRUOp, __nv_bfloat16>(pl, sp, stream);
    } else if (op == SGR_OP_MINGRU_LOG) {
        e = dtype == SGR_F32 ? dispatch<MinGRULogOp, float>(pl, sp, stream)
                             : dispatch<MinGRULogOp, __nv_bfloat16>(pl, sp, stream);
    } else {
        e = dtype == SGR_F32 ? dispatch<MinMaxOp, float>(pl, sp, stream)
                             : dispatch<MinMaxOp, __nv_bfloat16>(pl, sp, stream);
    }
    return e == cudaSuccess ? SGR_OK : SGR_ERR_CUDA;
}

// ---- gradients: the reverse-time tile kernel (scan_backward.cuh)
template <class BOp, typename IO, int V, int CG, int R>
cudaError_t launch_bwd_tile(const BwdParams &bp, cudaStream_t s) {
    if constexpr (R * V > 16) {
        return cudaErrorInvalidConfiguration;   // never planned (see make_plan)
    } else {
        // registers a data thread keeps live: four values per element, the
        // pair per channel and about 24 for addressing; blocks of 256 threads
        constexpr int NEED = 4 * R * V + 2 * V + 24;
        constexpr int MINB = NEED <= 56 ? 4 : (NEED <= 72 ? 3 : 2);
        auto kernel = scan_backward_kernel<BOp, IO, V, CG, R, kWarps, MINB>;
        int64_t grid = 0;
        const cudaError_t e = tile_grid(kernel, (kWarps + 1) * 32, bp.s.n_tiles, bp.s.ticket != nullptr, &grid);
        if (e != cudaSuccess) return e;
        kernel<<<unsigned(grid), (kWarps + 1) * 32, 0, s>>>(bp);
        return cudaGetLastError();
    }
}

template <class BOp, typename IO, int V, int CG>
cudaError_t dispatch_bwd_r(const Plan &pl, const BwdParams &bp, cudaStream_t s) {
    switch (pl.r) {
        case 1: return launch_bwd_tile<BOp, IO, V, CG, 1>(bp, s);
        case 2: return launch_bwd_tile<BOp, IO, V, CG, 2>(bp, s);
        case 4: return launch_bwd_tile<BOp, IO, V, CG, 4>(bp, s);
        default: return launch_bwd_tile<BOp, IO, V, CG, 8>(bp, s);
    }
}

// ---- channel-sequential gradient launch (wide batches)
template <class BOp, typename IO, bool DT>
cudaError_t launch_sequential_bwd_dt(const BwdParams &bp, const CUtensorMap (&m)[7], cudaStream_t s) {
    constexpr int WB = kSeqWarpsPerBlock;
    constexpr int CW = 32;
    constexpr int kRowBytes = seq_row_bytes<IO>();
    constexpr size_t kGap = DT ? kSeqGapBytes : 0;
    auto kernel = scan_sequential_backward_kernel<BOp, IO, WB, DT>;
    const ScanParams &sp = bp.s;
    SeqDev d;
    cudaError_t e =
        seq_device(reinterpret_cast<const void *>(kernel), seq_bwd_warp_bytes(kSeqMinSlots, kRowBytes, kGap), &d);
    if (e != cudaSuccess) return e;
    SeqBwdParams q;
    q.g = bp;
    q.n_groups = (sp.D + CW - 1) / CW;
    q.n_warps = sp.B * q.n_groups;
    const SeqLayout lay = seq_layout((q.n_warps + WB - 1) / WB * WB, kRowBytes, d.sms, size_t(d.smem_sm),
                                     size_t(d.reserved), size_t(d.smem_block), SEQ_BACKWARD, kGap);
    q.slots = lay.slots;
    const int64_t grid = (q.n_warps + WB - 1) / WB;
    kernel<<<dim3(unsigned(grid)), WB * 32, lay.smem, s>>>(q, m[0], m[1], m[2], m[3], m[4], m[5], m[6]);
    return cudaGetLastError();
}

template <class BOp, typename IO>
cudaError_t launch_sequential_bwd(const BwdParams &bp, cudaStream_t s) {
    constexpr int CW = 32;
    const ScanParams &sp = bp.s;
    const int esz = int(sizeof(IO));
    // k, hx (or r, s), dL/dh, the forward output, d in0, d in1, the gaps
    alignas(64) CUtensorMap m[7];
    if (!make_operand_map(&m[0], sp.in0, sp.B, sp.T, sp.D, esz, CW, kSeqRows) ||
        !make_operand_map(&m[1], sp.in1, sp.B, sp.T, sp.D, esz, CW, kSeqRows) ||
        !make_operand_map(&m[2], bp.gy, sp.B, sp.T, sp.D, esz, CW, kSeqRows) ||
        !make_operand_map(&m[3], bp.fwd, sp.B, sp.T, sp.D, esz, CW, kSeqRows) ||
        !make_operand_map(&m[4], sp.out, sp.B, sp.T, sp.D, esz, CW, kSeqRows) ||
        !make_operand_map(&m[5], bp.out1, sp.B, sp.T, sp.D, esz, CW, kSeqRows))
        return cudaErrorInvalidValue;
    if constexpr (BOp::kDecay) {
        if (make_seq_gap_map(&m[6], sp)) return launch_sequential_bwd_dt<BOp, IO, true>(bp, m, s);
    }
    m[6] = m[0];                              // not read without gaps through the copy engine
    return launch_sequential_bwd_dt<BOp, IO, false>(bp, m, s);
}

// whether a gradient of this shape walks whole sequences per warp
bool seq_backward_planned(int64_t B, int64_t T, int64_t D, int esz, bool aligned) {
    const int vw = 16 / esz;
    if (!aligned || D % vw != 0 || T > int64_t(std::numeric_limits<int>::max()) ||
        B > int64_t(std::numeric_limits<int>::max()))
        return false;
    const int ok = g_override_kind.load();
    if (seq_kind(ok)) return true;
    if (ok != KIND_AUTO) return false;
    const int64_t groups = B * ((D + 31) / 32);
    return groups >= int64_t(kSeqBwdMinWarpsPerSM) * kAssumedSMs;
}

// ---- pipelined gradient (narrow batches, aligned vector-width rows)
// fp32 32 channels x 2 rows per thread, bf16 64 channels x 4 rows per thread;
// 15 data warps + 1 carry warp, one block per SM, tiles of 120 rows (four
// operand boxes per ring slot, 3 slots: about 190 KB of shared memory), or 7
// data warps, two blocks per SM, tiles of 56 rows.  The plain gradients take
// the 15-warp blocks (fp32 B8 x 4096 x 1024: 140 against 150 us; MinMax
// B4 x 8192 x 768: 119 against 135 us).  The decayed one, whose longer phase
// A each block's carry warp waits behind, takes the 7-warp blocks where the
// channel tiles give the blocks in flight little look-back depth (fp32 B8 x
// 4096 x 1024, 256 chains: 187 against 195 us; bf16, 128 chains: 142
// against 150) and the 15-warp ones where the depth grows (fp32 B4 x 8192 x
// 768, 96 chains: 150 against 158 us).  The fp32 decayed gradient takes 4
// rows per thread (16 elements: the per-tile work is spread over twice the
// elements) in blocks of 6 data warps + 1 carry warp, two per SM (96-row
// tiles, a 2-slot ring of about 49 KB slots, 128 registers per thread):
// with 12 data warps per SM instead of 7 the latency each one exposes is
// hidden, measured 154.0 against 184.6 us for one 7-warp block per SM with
// 4 rows (override 2) on B8 x 4096 x 1024, 126.4 against 143.7 on
// B4 x 8192 x 768, 370.5 against 472.4 on B1 x 131072 x 512 (the 7-warp,
// 4-row blocks had measured 182.8 against 186.5 us for 2 rows and 193.1
// for 15-warp blocks on B8 x 4096 x 1024).  The plain fp32 gradients take
// the same blocks below 1.5 chains per SM (us, two 6-warp blocks against
// one 15-warp block, minGRU / MinMax): B4 x 8192 x 768 111.1 / 109.2
// against 119.3 / 116.2, B1 x 131072 x 512 307.7 / 301.7 against
// 371.2 / 361.1; at B8 x 4096 x 1024 (1.7 chains per SM) 143.3 / 143.8
// against 139.5 / 147.3.
template <typename IO, bool DECAY = false, int W = kPipeWarpsWide>
constexpr int bwd_pipe_r() {
    return (sizeof(IO) == 2 || W == kBwdPairWarps || (DECAY && W == kPipeWarps)) ? 4 : 2;
}
template <typename IO, bool DECAY, int W>
constexpr int bwd_pipe_minb() {
    return W == kBwdPairWarps || (W == kPipeWarps && !(sizeof(IO) == 4 && DECAY)) ? 2 : 1;
}
template <int W>
constexpr int bwd_pipe_stages() { return W == kBwdPairWarps ? kBwdPairStages : kStages; }
template <typename IO, bool DT = false, int W = kPipeWarpsWide, bool DECAY = false>
using BwdPipeShape = PipeBwdShape<IO, 4, pipe_cg<IO>(), bwd_pipe_r<IO, DECAY, W>(), bwd_pipe_stages<W>(), W, DT>;

// The gradient's tile plan: the pipelined kernel for aligned vector-width
// rows with at least two tiles per block (override 2 or 3 forces it wherever
// the rows allow), else the ticketed tile kernel (make_plan with force_tile).
// fp32 takes two 6-warp blocks per SM where that gives every block two
// tiles -- the decayed gradient at any chain count, the plain ones below 1.5
// chains of 32 channels per SM -- else (and under an override) the blocks
// below.
// decay: the time-decayed gradient.
Plan make_bwd_plan(int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype, bool aligned, bool decay = false) {
    const int esz = dtype == SGR_BF16 ? 2 : 4;
    const int vw = 16 / esz;
    const int ok = g_override_kind.load();
    const bool vec = aligned && D % vw == 0 && T < int64_t(std::numeric_limits<int>::max()) / 2;
    if (vec && (ok == KIND_AUTO || ok == KIND_PIPELINED || ok == KIND_PIPELINED_WIDE)) {
        Plan p;
        p.esz = esz;
        p.vec = true;
        p.kind = KIND_PIPELINED;
        p.V = 4;
        p.cg = esz == 4 ? 8 : 16;
        p.TC = p.cg * p.V;
        p.n_dt = (D + p.TC - 1) / p.TC;
        p.n_chains = B * p.n_dt;
        // tiles of `warps` data warps x (32 / cg) row groups x r rows
        auto shape = [&](int warps, int r, int stages, size_t smem) {
            p.warps = warps;
            p.r = r;
            p.stages = stages;
            p.smem = smem;
            p.TR = warps * (32 / p.cg) * r;
            p.n_chunks = (T + p.TR - 1) / p.TR;
            p.n_tiles = p.n_chains * p.n_chunks;
            p.off_words = 0;
            p.ws_bytes = 0;
            if (p.n_tiles > 0) {
                p.off_words = kAlign;
                p.ws_bytes = kAlign;
                if (p.n_chunks > 1) p.ws_bytes = align_up(p.off_words + size_t(p.n_tiles) * 3 * p.TC * 8, kAlign);
            }
        };
        const int64_t chains = B * ((D + (esz == 4 ? 32 : 64) - 1) / (esz == 4 ? 32 : 64));
        if (esz == 4 && ok == KIND_AUTO && (decay || 2 * chains < 3 * kAssumedSMs)) {
            shape(kBwdPairWarps, 4, kBwdPairStages, BwdPipeShape<float, false, kBwdPairWarps>::smem_bytes);
            if (p.n_tiles >= 4 * kAssumedSMs) return p;
        }
        // blocks of 15 data warps, one per SM, or of 7, two per SM (override
        // 2; bf16 decay with at least 0.8 chains per SM); the fp32 decayed
        // gradient with 7-warp blocks takes 4 rows per thread, one block per SM
        const bool narrow = ok == KIND_PIPELINED ||
                            (ok == KIND_AUTO && decay && (esz == 4 || 5 * chains >= 4 * kAssumedSMs));
        const int r = (esz == 2 || (decay && narrow)) ? 4 : 2;
        size_t smem;
        if (esz == 4)
            smem = narrow ? (decay ? BwdPipeShape<float, false, kPipeWarps, true>::smem_bytes
                                   : BwdPipeShape<float, false, kPipeWarps>::smem_bytes)
                          : BwdPipeShape<float>::smem_bytes;
        else
            smem = narrow ? BwdPipeShape<__nv_bfloat16, false, kPipeWarps>::smem_bytes
                          : BwdPipeShape<__nv_bfloat16>::smem_bytes;
        shape(narrow ? kPipeWarps : kPipeWarpsWide, r, kStages, smem);
        if (ok != KIND_AUTO || p.n_tiles >= 2 * kAssumedSMs) return p;
    }
    return make_plan(B, T, D, dtype, aligned, true);
}

template <class BOp, typename IO, bool DT, int W>
cudaError_t launch_pipelined_bwd_shape(const BwdParams &bp, const CUtensorMap (&m)[6], cudaStream_t s) {
    constexpr int CG = pipe_cg<IO>();
    constexpr int R = bwd_pipe_r<IO, BOp::kDecay, W>();
    using Shape = BwdPipeShape<IO, DT, W, BOp::kDecay>;
    auto kernel = scan_pipelined_backward_kernel<BOp, IO, 4, CG, R, bwd_pipe_stages<W>(), W,
                                                 bwd_pipe_minb<IO, BOp::kDecay, W>(), DT>;
    constexpr size_t smem = Shape::smem_bytes;
    constexpr int NT = (W + 1) * 32;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    // per-device one-time set-up of the shared-memory limit and occupancy
    static std::atomic<int> occ_cache[64];
    int occ = (dev >= 0 && dev < 64) ? occ_cache[dev].load() : 0;
    if (occ == 0) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, NT, smem);
        if (e != cudaSuccess) return e;
        if (occ <= 0) return cudaErrorInvalidConfiguration;
        if (dev >= 0 && dev < 64) occ_cache[dev].store(occ);
    }
    const DeviceInfo di = device_info(dev);
    if (di.sms <= 0) return cudaErrorInvalidDevice;
    const int64_t grid = std::min<int64_t>(bp.s.n_tiles, int64_t(di.sms) * occ);
    BwdParams args = bp;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args, m[0], m[1], m[2], m[3], m[4], m[5]);
}

template <class BOp, typename IO, int W>
cudaError_t launch_pipelined_bwd(const BwdParams &bp, cudaStream_t s) {
    using Shape = BwdPipeShape<IO, false, W, BOp::kDecay>;
    const ScanParams &sp = bp.s;
    const int esz = int(sizeof(IO));
    // k, hx (or r, s), dL/dh, the forward output; the decay's gaps and rates
    alignas(64) CUtensorMap m[6];
    if (!make_operand_map(&m[0], sp.in0, sp.B, sp.T, sp.D, esz, Shape::TC, Shape::TR) ||
        !make_operand_map(&m[1], sp.in1, sp.B, sp.T, sp.D, esz, Shape::TC, Shape::TR) ||
        !make_operand_map(&m[2], bp.gy, sp.B, sp.T, sp.D, esz, Shape::TC, Shape::TR) ||
        !make_operand_map(&m[3], bp.fwd, sp.B, sp.T, sp.D, esz, Shape::TC, Shape::TR))
        return cudaErrorInvalidValue;
    if constexpr (BOp::kDecay && BwdPipeShape<IO, true, W, true>::dec_boxable) {
        if (make_decay_maps(&m[4], &m[5], sp, Shape::TR, Shape::TC))
            return launch_pipelined_bwd_shape<BOp, IO, true, W>(bp, m, s);
    }
    m[4] = m[0];                              // not read without decay operands through the copy engine
    m[5] = m[0];
    return launch_pipelined_bwd_shape<BOp, IO, false, W>(bp, m, s);
}

template <class BOp, typename IO>
cudaError_t dispatch_bwd(const Plan &pl, const BwdParams &bp, cudaStream_t s) {
    constexpr int VW = 16 / int(sizeof(IO));
    if (pl.kind == KIND_PIPELINED) {
        if constexpr (sizeof(IO) == 4) {
            if (pl.warps == kBwdPairWarps) return launch_pipelined_bwd<BOp, IO, kBwdPairWarps>(bp, s);
        }
        return pl.warps == kPipeWarps ? launch_pipelined_bwd<BOp, IO, kPipeWarps>(bp, s)
                                      : launch_pipelined_bwd<BOp, IO, kPipeWarpsWide>(bp, s);
    }
    if (!pl.vec) return dispatch_bwd_r<BOp, IO, 1, 32>(pl, bp, s);
    return dispatch_bwd_r<BOp, IO, VW, 8>(pl, bp, s);
}

sgr_status_t run_scan_backward(sgr_op_t op, const void *in0, const void *in1, const void *init,
                               int64_t init_bs, const void *fwd, const void *gy, void *out0,
                               void *out1, void *dinit, int64_t dinit_bs, int64_t B, int64_t T,
                               int64_t D, sgr_dtype_t dtype, void *ws, size_t ws_bytes,
                               cudaStream_t stream, const DecayArgs *dec = nullptr,
                               float *dlam = nullptr) {
    if (dtype != SGR_F32 && dtype != SGR_BF16) return SGR_ERR_INVALID_ARG;
    if (op != SGR_OP_MINGRU && op != SGR_OP_MINMAX) return SGR_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || D < 0 || init_bs < 0 || dinit_bs < 0) return SGR_ERR_INVALID_ARG;
    if (B == 0 || D == 0) {
        // no elements: dL/dlambda is zero
        if (dec && dlam && D > 0 && cudaMemsetAsync(dlam, 0, size_t(D) * sizeof(float), stream) != cudaSuccess)
            return SGR_ERR_CUDA;
        return SGR_OK;
    }
    if (dinit && B > 1 && dinit_bs < D) return SGR_ERR_INVALID_ARG;   // rows would overlap
    const int esz = dtype == SGR_BF16 ? 2 : 4;
    int64_t n = 0, nbytes = 0, tmp = 0;
    if (!mul_ok(B, T, &n) || !mul_ok(n, D, &n) || !mul_ok(n, esz, &nbytes)) return SGR_ERR_UNSUPPORTED;
    for (int64_t bs : {init_bs, dinit_bs})
        if (!mul_ok(B - 1, bs, &tmp) || !mul_ok(tmp + D, esz, &tmp)) return SGR_ERR_UNSUPPORTED;
    const size_t db = dinit ? rows_span(B, D, dinit_bs, esz) : 0;
    if (T == 0) {
        // no steps: the gradients reaching the initial state and lambda are zero
        if (dec && dlam && cudaMemsetAsync(dlam, 0, size_t(D) * sizeof(float), stream) != cudaSuccess)
            return SGR_ERR_CUDA;
        if (dinit) {
            if (dinit_bs == D || B == 1) {
                if (cudaMemsetAsync(dinit, 0, size_t(D) * esz * (B == 1 ? 1 : B), stream) != cudaSuccess)
                    return SGR_ERR_CUDA;
            } else if (cudaMemset2DAsync(dinit, size_t(dinit_bs) * esz, 0, size_t(D) * esz, size_t(B),
                                         stream) != cudaSuccess) {
                return SGR_ERR_CUDA;
            }
        }
        return SGR_OK;
    }
    if (!in0 || !in1 || !fwd || !gy || !out0 || !out1) return SGR_ERR_INVALID_ARG;
    const sgr_status_t dst = check_decay(dec, B, T, D);
    if (dst != SGR_OK) return dst;
    const size_t tb = size_t(nbytes);
    const size_t ib = init ? rows_span(B, D, init_bs, esz) : 0;
    const void *ins[5] = {in0, in1, fwd, gy, init};
    const size_t in_bytes[5] = {tb, tb, tb, tb, ib};
    for (int i = 0; i < 5; ++i) {
        if (overlaps(out0, tb, ins[i], in_bytes[i]) || overlaps(out1, tb, ins[i], in_bytes[i]) ||
            overlaps(dinit, db, ins[i], in_bytes[i]))
            return SGR_ERR_INVALID_ARG;
    }
    if (overlaps(out0, tb, out1, tb) || overlaps(out0, tb, dinit, db) || overlaps(out1, tb, dinit, db))
        return SGR_ERR_INVALID_ARG;
    if (overlaps_decay(dec, out0, tb, B, T, D) || overlaps_decay(dec, out1, tb, B, T, D) ||
        overlaps_decay(dec, dinit, db, B, T, D))
        return SGR_ERR_INVALID_ARG;
    if (dec && dlam) {
        // dL/dlambda is cleared and accumulated while everything else is read
        // or written: it shares memory with none of it
        const size_t lb = decay_lam_bytes(D);
        if (overlaps_decay(dec, dlam, lb, B, T, D) || overlaps(dlam, lb, out0, tb) ||
            overlaps(dlam, lb, out1, tb) || overlaps(dlam, lb, dinit, db))
            return SGR_ERR_INVALID_ARG;
        for (int i = 0; i < 5; ++i)
            if (overlaps(dlam, lb, ins[i], in_bytes[i])) return SGR_ERR_INVALID_ARG;
    }

    const bool aligned = aligned16(in0) && aligned16(in1) && aligned16(fwd) && aligned16(gy) &&
                         aligned16(out0) && aligned16(out1);
    const bool seq = seq_backward_planned(B, T, D, esz, aligned);
    const Plan pl = make_bwd_plan(B, T, D, dtype, aligned, dec != nullptr);
    if (!seq && pl.n_tiles > int64_t(std::numeric_limits<int>::max())) return SGR_ERR_UNSUPPORTED;

    BwdParams bp;
    std::memset(&bp, 0, sizeof(bp));
    ScanParams &sp = bp.s;
    sp.in0 = in0; sp.in1 = in1; sp.init = nullptr; sp.init_bs = 0; sp.out = out0;
    sp.B = B; sp.T = T; sp.D = D;
    sp.n_dt = pl.n_dt; sp.n_chains = pl.n_chains; sp.n_chunks = pl.n_chunks; sp.n_tiles = pl.n_tiles;
    sp.by_chains = make_fastdiv(uint32_t(pl.n_chains));
    sp.by_dt = make_fastdiv(uint32_t(pl.n_dt));
    sp.epoch = 0;
    sp.spin_limit = g_spin_limit.load();
    sp.drop_tile = g_drop_tile.load();
    bp.fwd = fwd; bp.gy = gy; bp.init = init; bp.init_bs = init_bs;
    bp.out1 = out1; bp.dinit = dinit; bp.dinit_bs = dinit_bs;
    set_decay(sp, dec);
    bp.dlam = dec ? dlam : nullptr;
    if (seq) {
        // one warp per channel group over the whole sequence: no hand-off
        // words; the workspace header receives the status word
        if (!ws || ws_bytes < kAlign || !aligned16(ws)) return SGR_ERR_WORKSPACE;
        sp.status = static_cast<uint32_t *>(ws);
        if (bp.dlam && cudaMemsetAsync(bp.dlam, 0, size_t(D) * sizeof(float), stream) != cudaSuccess)
            return SGR_ERR_CUDA;
        cudaError_t e;
        if (op == SGR_OP_MINGRU && dec) {
            e = dtype == SGR_F32 ? launch_sequential_bwd<MinGRUDecayBwd, float>(bp, stream)
                                 : launch_sequential_bwd<MinGRUDecayBwd, __nv_bfloat16>(bp, stream);
        } else if (op == SGR_OP_MINGRU) {
            e = dtype == SGR_F32 ? launch_sequential_bwd<MinGRUBwd, float>(bp, stream)
                                 : launch_sequential_bwd<MinGRUBwd, __nv_bfloat16>(bp, stream);
        } else {
            e = dtype == SGR_F32 ? launch_sequential_bwd<MinMaxBwd, float>(bp, stream)
                                 : launch_sequential_bwd<MinMaxBwd, __nv_bfloat16>(bp, stream);
        }
        return e == cudaSuccess ? SGR_OK : SGR_ERR_CUDA;
    }
    if (!ws || ws_bytes < pl.ws_bytes || !aligned16(ws)) return SGR_ERR_WORKSPACE;
    sp.status = static_cast<uint32_t *>(ws);
    if (pl.n_chunks > 1) {
        char *w = static_cast<char *>(ws);
        sp.words = reinterpret_cast<uint64_t *>(w + pl.off_words);
        if (pl.kind == KIND_TILE) {
            // tile kernel: tiles go out by ticket in block start order
            sp.ticket = reinterpret_cast<uint32_t *>(w + kTicketOffset);
            if (cudaMemsetAsync(sp.ticket, 0, sizeof(uint32_t), stream) != cudaSuccess) return SGR_ERR_CUDA;
        }
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return SGR_ERR_CUDA;
        if (cs == cudaStreamCaptureStatusActive) {
            if (cudaMemsetAsync(sp.words, 0, pl.ws_bytes - pl.off_words, stream) != cudaSuccess)
                return SGR_ERR_CUDA;
            sp.epoch = 1;
        } else {
            sp.epoch = next_epoch();
        }
    }
    // dL/dlambda accumulates over the tiles with atomic adds
    if (bp.dlam && cudaMemsetAsync(bp.dlam, 0, size_t(D) * sizeof(float), stream) != cudaSuccess)
        return SGR_ERR_CUDA;
    cudaError_t e;
    if (op == SGR_OP_MINGRU && dec) {
        e = dtype == SGR_F32 ? dispatch_bwd<MinGRUDecayBwd, float>(pl, bp, stream)
                             : dispatch_bwd<MinGRUDecayBwd, __nv_bfloat16>(pl, bp, stream);
    } else if (op == SGR_OP_MINGRU) {
        e = dtype == SGR_F32 ? dispatch_bwd<MinGRUBwd, float>(pl, bp, stream)
                             : dispatch_bwd<MinGRUBwd, __nv_bfloat16>(pl, bp, stream);
    } else {
        e = dtype == SGR_F32 ? dispatch_bwd<MinMaxBwd, float>(pl, bp, stream)
                             : dispatch_bwd<MinMaxBwd, __nv_bfloat16>(pl, bp, stream);
    }
    return e == cudaSuccess ? SGR_OK : SGR_ERR_CUDA;
}

// ---- sequence summaries (time axis split across devices)
struct SumPlan {
    int V = 1;
    int64_t seg = 0, n_seg = 0;
    size_t ws = 0;
    bool seq = false;     // warps folding TMA-fed segments of 32-channel groups
};

// Aligned vector-width rows: one warp per (segment, 32-channel group),
// segments whole 16-row slots (at most 512 of them), about 52 warps per SM in
// all (several waves of short segments; measured against 13-156 on the
// summary rows: 13 per SM in one wave was best for fp32 B8 x 4096 x 1024 by
// 2% but 20% slower for bf16 B16 x 2048 x 4096, more than 52 slower for the
// former).  Otherwise one thread per vector (or channel) per segment.
SumPlan make_sum_plan(int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype, bool aligned) {
    SumPlan sp;
    const int vw = dtype == SGR_BF16 ? 8 : 4;
    if (aligned && D % vw == 0 && T <= int64_t(std::numeric_limits<int>::max()) &&
        B <= int64_t(std::numeric_limits<int>::max())) {
        sp.seq = true;
        const int64_t chains = B * ((D + 31) / 32);
        const int64_t target = int64_t(52) * kAssumedSMs;
        const int64_t max_seg = std::min<int64_t>(512, (T + kSeqRows - 1) / kSeqRows);
        const int64_t n_seg = std::max<int64_t>(1, std::min<int64_t>((target + chains - 1) / chains, max_seg));
        sp.seg = ((T + n_seg - 1) / n_seg + kSeqRows - 1) / kSeqRows * kSeqRows;
        sp.n_seg = (T + sp.seg - 1) / sp.seg;
        const int64_t n_mid = sp.n_seg > 32 ? (sp.n_seg + 31) / 32 : 0;
        sp.ws = kAlign + align_up(size_t(sp.n_seg + n_mid) * size_t(B) * size_t(D) * sizeof(float2), kAlign);
        return sp;
    }
    // one 16-byte vector of channels per thread (4 fp32, 8 bf16)
    sp.V = (aligned && D % vw == 0) ? vw : 1;
    const int64_t groups = (D + sp.V - 1) / sp.V;
    // about 4096 threads per SM (two waves), each with rows of loads in flight, and at
    // most 512 segments so that the second pass (one thread per channel
    // folding its segments) stays short
    const int64_t target = int64_t(kAssumedSMs) * 4096;
    int64_t n_seg = (target + B * groups - 1) / (B * groups);
    n_seg = std::max<int64_t>(1, std::min<int64_t>({n_seg, (T + 7) / 8, int64_t(512)}));
    sp.seg = (T + n_seg - 1) / n_seg;
    sp.n_seg = (T + sp.seg - 1) / sp.seg;
    // the status word's header, the partials, then (more than 32 segments)
    // their folds in groups of 32
    const int64_t n_mid = sp.n_seg > 32 ? (sp.n_seg + 31) / 32 : 0;
    sp.ws = kAlign + align_up(size_t(sp.n_seg + n_mid) * size_t(B) * size_t(D) * sizeof(float2), kAlign);
    return sp;
}

// pass 1 on TMA-fed warps: one per (segment, 32-channel group)
template <class Op, typename IO>
cudaError_t launch_sequential_fold(const SumPlan &pl, const ScanParams &sp, float2 *partial, cudaStream_t s) {
    constexpr int WB = kSeqWarpsPerBlock;
    constexpr int CW = 32;
    constexpr int kRowBytes = seq_row_bytes<IO>();
    auto kernel = scan_sequential_fold_kernel<Op, IO, WB>;
    alignas(64) CUtensorMap map0, map1;
    if (!make_operand_map(&map0, sp.in0, sp.B, sp.T, sp.D, int(sizeof(IO)), CW, kSeqRows) ||
        !make_operand_map(&map1, sp.in1, sp.B, sp.T, sp.D, int(sizeof(IO)), CW, kSeqRows))
        return cudaErrorInvalidValue;
    SeqDev d;
    cudaError_t e = seq_device(reinterpret_cast<const void *>(kernel), seq_fold_warp_bytes(kSeqMinSlots, kRowBytes), &d);
    if (e != cudaSuccess) return e;
    SeqFoldParams q;
    q.s = sp;
    q.n_groups = (sp.D + CW - 1) / CW;
    q.n_warps = pl.n_seg * sp.B * q.n_groups;
    q.seg_rows = pl.seg;
    q.partial = partial;
    const SeqLayout lay = seq_layout((q.n_warps + WB - 1) / WB * WB, kRowBytes, d.sms, size_t(d.smem_sm),
                                     size_t(d.reserved), size_t(d.smem_block), SEQ_FOLD);
    q.slots = lay.slots;
    kernel<<<dim3(unsigned((q.n_warps + WB - 1) / WB)), WB * 32, lay.smem, s>>>(q, map0, map1);
    return cudaGetLastError();
}

template <class Op, typename IO>
cudaError_t launch_summary(const SumPlan &pl, const ScanParams &sp, float2 *partial, float2 *out,
                           cudaStream_t s) {
    constexpr int VW = 16 / int(sizeof(IO));
    if (pl.seq) {
        const cudaError_t e = launch_sequential_fold<Op, IO>(pl, sp, partial, s);
        if (e != cudaSuccess) return e;
    } else {
        const int64_t groups = (sp.D + pl.V - 1) / pl.V;
        const int64_t n = sp.B * groups * pl.n_seg;
        const unsigned grid = unsigned(std::min<int64_t>((n + 255) / 256, int64_t(kAssumedSMs) * 16));
        if (pl.V == 1) {
            scan_summary_kernel<Op, IO, 1><<<grid, 256, 0, s>>>(sp, pl.seg, pl.n_seg, partial);
        } else {
            scan_summary_kernel<Op, IO, VW><<<grid, 256, 0, s>>>(sp, pl.seg, pl.n_seg, partial);
        }
    }
    const int64_t BD = sp.B * sp.D;
    auto grid_for = [](int64_t n) { return unsigned(std::min<int64_t>((n + 255) / 256, int64_t(kAssumedSMs) * 16)); };
    if (pl.n_seg > 32) {
        // two levels, so no thread folds more than 32 pairs in a row
        const int64_t n_mid = (pl.n_seg + 31) / 32;
        float2 *mid = partial + pl.n_seg * BD;
        fold_partials_kernel<Op><<<grid_for(n_mid * BD), 256, 0, s>>>(partial, pl.n_seg, 32, BD, mid);
        fold_partials_kernel<Op><<<grid_for(BD), 256, 0, s>>>(mid, n_mid, n_mid, BD, out);
    } else {
        fold_partials_kernel<Op><<<grid_for(BD), 256, 0, s>>>(partial, pl.n_seg, pl.n_seg > 0 ? pl.n_seg : 1,
                                                              BD, out);
    }
    return cudaGetLastError();
}

// ---- input projection fused with the scan (projected_scan.cuh)
size_t projected_ws_bytes(int64_t B, int64_t T, int64_t D) {
    const int64_t n_chunks = (T + proj::kTR - 1) / proj::kTR;
    const int64_t n_tiles = n_chunks * B * (D / proj::kTC);
    return align_up(kAlign + size_t(n_tiles) * 3 * proj::kTC * 8, kAlign);
}

sgr_status_t run_projected_scan(const void *x, const void *w, const float *h0, int64_t h0_bs, float *h,
                                int64_t B, int64_t T, int64_t D, int64_t d_in, void *ws, size_t ws_bytes,
                                cudaStream_t stream) {
    if (B < 0 || T < 0 || D < 0 || d_in < 0 || h0_bs < 0) return SGR_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || D == 0) return SGR_OK;
    if (D % proj::kTC != 0 || d_in % proj::kKB != 0 || d_in == 0) return SGR_ERR_UNSUPPORTED;
    if (!x || !w || !h) return SGR_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w)) return SGR_ERR_INVALID_ARG;
    int64_t n = 0, xb = 0, hb = 0, wb = 0, tmp = 0;
    if (!mul_ok(B, T, &n) || !mul_ok(n, d_in, &xb) || !mul_ok(xb, 2, &xb)) return SGR_ERR_UNSUPPORTED;
    if (!mul_ok(n, D, &hb) || !mul_ok(hb, 4, &hb)) return SGR_ERR_UNSUPPORTED;
    if (!mul_ok(2 * D, d_in, &wb) || !mul_ok(wb, 2, &wb)) return SGR_ERR_UNSUPPORTED;
    if (h0 && (!mul_ok(B - 1, h0_bs, &tmp) || !mul_ok(tmp + D, 4, &tmp))) return SGR_ERR_UNSUPPORTED;
    if (T > (int64_t(1) << 31) - 1 || d_in > (int64_t(1) << 31) - 1 || 2 * D > (int64_t(1) << 31) - 1)
        return SGR_ERR_UNSUPPORTED;                    // tensor-map coordinates are 32-bit
    const size_t ib = h0 ? rows_span(B, D, h0_bs, 4) : 0;
    if (overlaps(h, size_t(hb), x, size_t(xb)) || overlaps(h, size_t(hb), w, size_t(wb)) ||
        overlaps(h, size_t(hb), h0, ib))
        return SGR_ERR_INVALID_ARG;
    const int64_t n_chunks = (T + proj::kTR - 1) / proj::kTR;
    const int64_t n_dt = D / proj::kTC;
    const int64_t n_tiles = n_chunks * B * n_dt;
    if (n_tiles > int64_t(std::numeric_limits<int>::max())) return SGR_ERR_UNSUPPORTED;
    const size_t need = projected_ws_bytes(B, T, D);
    if (!ws || ws_bytes < need || !aligned16(ws)) return SGR_ERR_WORKSPACE;

    ProjParams pp;
    std::memset(&pp, 0, sizeof(pp));
    ScanParams &sp = pp.s;
    sp.init = h0; sp.init_bs = h0_bs; sp.out = h;
    sp.B = B; sp.T = T; sp.D = D;
    sp.n_dt = n_dt; sp.n_chains = B * n_dt; sp.n_chunks = n_chunks; sp.n_tiles = n_tiles;
    sp.by_chains = make_fastdiv(uint32_t(sp.n_chains));
    sp.by_dt = make_fastdiv(uint32_t(n_dt));
    sp.spin_limit = g_spin_limit.load();
    sp.drop_tile = g_drop_tile.load();
    char *wsc = static_cast<char *>(ws);
    sp.status = reinterpret_cast<uint32_t *>(wsc);
    sp.words = reinterpret_cast<uint64_t *>(wsc + kAlign);
    pp.d_in = d_in;

    EncodeTiledFn enc = encode_tiled_fn();
    if (enc == nullptr) return SGR_ERR_CUDA;
    alignas(64) CUtensorMap map_x, map_w;
    {
        const cuuint64_t dims[3] = {cuuint64_t(d_in), cuuint64_t(T), cuuint64_t(B)};
        const cuuint64_t strides[2] = {cuuint64_t(d_in) * 2, cuuint64_t(T) * cuuint64_t(d_in) * 2};
        const cuuint32_t box[3] = {cuuint32_t(proj::kKB), cuuint32_t(proj::kTR), 1u};
        const cuuint32_t es[3] = {1u, 1u, 1u};
        if (enc(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(x), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return SGR_ERR_CUDA;
    }
    {
        // W (2 D, d_in) as (d_in, 16 rows of a group, k/hx, D / 16 groups)
        const cuuint64_t dims[4] = {cuuint64_t(d_in), cuuint64_t(proj::kGrp), 2, cuuint64_t(D / proj::kGrp)};
        const cuuint64_t strides[3] = {cuuint64_t(d_in) * 2, cuuint64_t(D) * cuuint64_t(d_in) * 2,
                                       cuuint64_t(proj::kGrp) * cuuint64_t(d_in) * 2};
        const cuuint32_t box[4] = {cuuint32_t(proj::kKB), cuuint32_t(proj::kGrp), 2u,
                                   cuuint32_t(proj::kTC / proj::kGrp)};
        const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
        if (enc(&map_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(w), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return SGR_ERR_CUDA;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return SGR_ERR_CUDA;
    if (cs == cudaStreamCaptureStatusActive) {
        if (cudaMemsetAsync(sp.words, 0, need - kAlign, stream) != cudaSuccess) return SGR_ERR_CUDA;
        sp.epoch = 1;
    } else {
        sp.epoch = next_epoch();
    }
    // persistent blocks, as many as are resident at once (one per SM: the
    // block holds all 512 tensor-memory columns), launched cooperatively so
    // that every look-back waits for a block that is running
    static std::atomic<int> occ_cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SGR_ERR_CUDA;
    int occ = (dev >= 0 && dev < 64) ? occ_cache[dev].load() : 0;
    if (occ == 0) {
        if (cudaFuncSetAttribute(mingru_projected_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(proj::kSmemBytes)) != cudaSuccess)
            return SGR_ERR_CUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, mingru_projected_scan_kernel, proj::kThreads,
                                                          proj::kSmemBytes) != cudaSuccess)
            return SGR_ERR_CUDA;
        if (occ <= 0) return SGR_ERR_UNSUPPORTED;
        occ = 1;                                       // tensor memory: one block per SM whatever fits
        if (dev >= 0 && dev < 64) occ_cache[dev].store(occ);
    }
    const DeviceInfo di = device_info(dev);
    if (di.sms <= 0) return SGR_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(std::min<int64_t>(n_tiles, int64_t(di.sms) * occ)));
    cfg.blockDim = dim3(proj::kThreads);
    cfg.dynamicSmemBytes = proj::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mingru_projected_scan_kernel, pp, map_x, map_w) != cudaSuccess)
        return SGR_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SGR_OK : SGR_ERR_CUDA;
}

}  // namespace

extern "C" {

sgr_status_t mingru_scan(const void *k, const void *hx, const void *h0, int64_t h0_batch_stride,
                         void *h, int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype,
                         void *workspace, size_t ws_bytes, cudaStream_t stream) {
    return run_scan(SGR_OP_MINGRU, k, hx, h0, h0_batch_stride, h, B, T, D, dtype, workspace,
                    ws_bytes, stream);
}

sgr_status_t mingru_scan_log(const void *k, const void *hx, const void *h0, int64_t h0_batch_stride,
                             void *h, int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype,
                             void *workspace, size_t ws_bytes, cudaStream_t stream) {
    return run_scan(SGR_OP_MINGRU_LOG, k, hx, h0, h0_batch_stride, h, B, T, D, dtype, workspace,
                    ws_bytes, stream);
}

sgr_status_t minmax_scan(const void *r, const void *s, const void *x0, int64_t x0_batch_stride,
                         void *x, int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype,
                         void *workspace, size_t ws_bytes, cudaStream_t stream) {
    return run_scan(SGR_OP_MINMAX, r, s, x0, x0_batch_stride, x, B, T, D, dtype, workspace,
                    ws_bytes, stream);
}

sgr_status_t mingru_step(const void *k_t, int64_t k_bs, const void *hx_t, int64_t hx_bs,
                         const void *h_prev, int64_t hp_bs, void *h_out, int64_t ho_bs,
                         int64_t B, int64_t D, sgr_dtype_t dtype, cudaStream_t stream) {
    if (dtype != SGR_F32 && dtype != SGR_BF16) return SGR_ERR_INVALID_ARG;
    if (B < 0 || D < 0 || k_bs < 0 || hx_bs < 0 || hp_bs < 0 || ho_bs < 0) return SGR_ERR_INVALID_ARG;
    if (B == 0 || D == 0) return SGR_OK;
    if (!k_t || !hx_t || !h_out) return SGR_ERR_INVALID_ARG;
    if (B > 1 && ho_bs < D) return SGR_ERR_INVALID_ARG;   // output rows would overlap
    const int esz = dtype == SGR_BF16 ? 2 : 4;
    int64_t tmp = 0;
    for (int64_t bs : {k_bs, hx_bs, hp_bs, ho_bs})
        if (!mul_ok(B - 1, bs, &tmp) || !mul_ok(tmp + D, esz, &tmp)) return SGR_ERR_UNSUPPORTED;
    const size_t ob = rows_span(B, D, ho_bs, esz);
    if (overlaps(h_out, ob, k_t, rows_span(B, D, k_bs, esz)) ||
        overlaps(h_out, ob, hx_t, rows_span(B, D, hx_bs, esz)))
        return SGR_ERR_INVALID_ARG;
    const bool in_place = (h_prev == h_out) && (hp_bs == ho_bs);
    if (h_prev && !in_place && overlaps(h_out, ob, h_prev, rows_span(B, D, hp_bs, esz)))
        return SGR_ERR_INVALID_ARG;
    const int64_t n = B * D;
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 16);
    if (dtype == SGR_F32) {
        mingru_step_kernel<float><<<unsigned(blocks), 256, 0, stream>>>(
            static_cast<const float *>(k_t), k_bs, static_cast<const float *>(hx_t), hx_bs,
            static_cast<const float *>(h_prev), hp_bs, static_cast<float *>(h_out), ho_bs, B, D);
    } else {
        mingru_step_kernel<__nv_bfloat16><<<unsigned(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(k_t), k_bs,
            static_cast<const __nv_bfloat16 *>(hx_t), hx_bs,
            static_cast<const __nv_bfloat16 *>(h_prev), hp_bs,
            static_cast<__nv_bfloat16 *>(h_out), ho_bs, B, D);
    }
    return cudaGetLastError() == cudaSuccess ? SGR_OK : SGR_ERR_CUDA;
}

sgr_status_t mingru_scan_backward(const void *k, const void *hx, const void *h0,
                                  int64_t h0_batch_stride, const void *h, const void *dh, void *dk,
                                  void *dhx, void *dh0, int64_t dh0_batch_stride, int64_t B,
                                  int64_t T, int64_t D, sgr_dtype_t dtype, void *workspace,
                                  size_t ws_bytes, cudaStream_t stream) {
    return run_scan_backward(SGR_OP_MINGRU, k, hx, h0, h0_batch_stride, h, dh, dk, dhx, dh0,
                             dh0_batch_stride, B, T, D, dtype, workspace, ws_bytes, stream);
}

sgr_status_t minmax_scan_backward(const void *r, const void *s, const void *x0,
                                  int64_t x0_batch_stride, const void *x, const void *dx, void *dr,
                                  void *ds, void *dx0, int64_t dx0_batch_stride, int64_t B,
                                  int64_t T, int64_t D, sgr_dtype_t dtype, void *workspace,
                                  size_t ws_bytes, cudaStream_t stream) {
    return run_scan_backward(SGR_OP_MINMAX, r, s, x0, x0_batch_stride, x, dx, dr, ds, dx0,
                             dx0_batch_stride, B, T, D, dtype, workspace, ws_bytes, stream);
}

sgr_status_t mingru_scan_decay(const void *k, const void *hx, const void *h0, int64_t h0_batch_stride,
                               const float *delta_t, int64_t delta_t_batch_stride, const float *lambda,
                               int log1p_delta, void *h, int64_t B, int64_t T, int64_t D,
                               sgr_dtype_t dtype, void *workspace, size_t ws_bytes, cudaStream_t stream) {
    DecayArgs dec;
    dec.dt = delta_t; dec.dt_bs = delta_t_batch_stride; dec.lam = lambda; dec.log1p = log1p_delta;
    return run_scan(SGR_OP_MINGRU, k, hx, h0, h0_batch_stride, h, B, T, D, dtype, workspace,
                    ws_bytes, stream, &dec);
}

sgr_status_t mingru_scan_decay_backward(const void *k, const void *hx, const void *h0,
                                        int64_t h0_batch_stride, const float *delta_t,
                                        int64_t delta_t_batch_stride, const float *lambda,
                                        int log1p_delta, const void *h, const void *dh, void *dk,
                                        void *dhx, void *dh0, int64_t dh0_batch_stride,
                                        float *dlambda, int64_t B, int64_t T, int64_t D,
                                        sgr_dtype_t dtype, void *workspace, size_t ws_bytes,
                                        cudaStream_t stream) {
    DecayArgs dec;
    dec.dt = delta_t; dec.dt_bs = delta_t_batch_stride; dec.lam = lambda; dec.log1p = log1p_delta;
    return run_scan_backward(SGR_OP_MINGRU, k, hx, h0, h0_batch_stride, h, dh, dk, dhx, dh0,
                             dh0_batch_stride, B, T, D, dtype, workspace, ws_bytes, stream, &dec,
                             dlambda);
}

size_t sgr_projected_workspace_size(int64_t B, int64_t T, int64_t D) {
    if (B <= 0 || T <= 0 || D <= 0 || D % proj::kTC != 0) return 0;
    return projected_ws_bytes(B, T, D);
}

sgr_status_t mingru_projected_scan(const void *x, const void *w, const float *h0, int64_t h0_batch_stride,
                                   float *h, int64_t B, int64_t T, int64_t D, int64_t d_in,
                                   void *workspace, size_t ws_bytes, cudaStream_t stream) {
    return run_projected_scan(x, w, h0, h0_batch_stride, h, B, T, D, d_in, workspace, ws_bytes, stream);
}

size_t sgr_summary_workspace_size(int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype) {
    if (dtype != SGR_F32 && dtype != SGR_BF16) return 0;
    if (B <= 0 || T <= 0 || D <= 0) return 0;
    const SumPlan a = make_sum_plan(B, T, D, dtype, true), b = make_sum_plan(B, T, D, dtype, false);
    return a.ws > b.ws ? a.ws : b.ws;
}

sgr_status_t sgr_scan_summary(sgr_op_t op, const void *in0, const void *in1, int64_t B, int64_t T,
                              int64_t D, sgr_dtype_t dtype, float *pairs, void *workspace,
                              size_t ws_bytes, cudaStream_t stream) {
    if (dtype != SGR_F32 && dtype != SGR_BF16) return SGR_ERR_INVALID_ARG;
    if (op != SGR_OP_MINGRU && op != SGR_OP_MINMAX) return SGR_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || D < 0) return SGR_ERR_INVALID_ARG;
    if (B == 0 || D == 0) return SGR_OK;
    if (!pairs) return SGR_ERR_INVALID_ARG;
    const int esz = dtype == SGR_BF16 ? 2 : 4;
    int64_t n = 0, nbytes = 0;
    if (!mul_ok(B, T, &n) || !mul_ok(n, D, &n) || !mul_ok(n, esz, &nbytes)) return SGR_ERR_UNSUPPORTED;
    const size_t pb = size_t(B) * size_t(D) * 2 * sizeof(float);
    if (T == 0) {
        // no steps: the identity pair (minGRU (1, 0); MinMax (+inf, -inf))
        const int64_t BD = B * D;
        const unsigned g = unsigned(std::min<int64_t>((BD + 255) / 256, int64_t(kAssumedSMs) * 16));
        float2 *out = reinterpret_cast<float2 *>(pairs);
        if (op == SGR_OP_MINGRU) fold_partials_kernel<MinGRUOp><<<g, 256, 0, stream>>>(nullptr, 0, 1, BD, out);
        else fold_partials_kernel<MinMaxOp><<<g, 256, 0, stream>>>(nullptr, 0, 1, BD, out);
        return cudaGetLastError() == cudaSuccess ? SGR_OK : SGR_ERR_CUDA;
    }
    if (!in0 || !in1) return SGR_ERR_INVALID_ARG;
    if (overlaps(pairs, pb, in0, size_t(nbytes)) || overlaps(pairs, pb, in1, size_t(nbytes)))
        return SGR_ERR_INVALID_ARG;
    const bool aligned = aligned16(in0) && aligned16(in1);
    const SumPlan pl = make_sum_plan(B, T, D, dtype, aligned);
    if (!workspace || ws_bytes < pl.ws || !aligned16(workspace)) return SGR_ERR_WORKSPACE;
    if (overlaps(workspace, pl.ws, pairs, pb)) return SGR_ERR_INVALID_ARG;
    ScanParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.in0 = in0; sp.in1 = in1; sp.B = B; sp.T = T; sp.D = D;
    sp.status = static_cast<uint32_t *>(workspace);                  // header: the status word
    float2 *partial = reinterpret_cast<float2 *>(static_cast<char *>(workspace) + kAlign);
    float2 *out = reinterpret_cast<float2 *>(pairs);
    cudaError_t e;
    if (op == SGR_OP_MINGRU) {
        e = dtype == SGR_F32 ? launch_summary<MinGRUOp, float>(pl, sp, partial, out, stream)
                             : launch_summary<MinGRUOp, __nv_bfloat16>(pl, sp, partial, out, stream);
    } else {
        e = dtype == SGR_F32 ? launch_summary<MinMaxOp, float>(pl, sp, partial, out, stream)
                             : launch_summary<MinMaxOp, __nv_bfloat16>(pl, sp, partial, out, stream);
    }
    return e == cudaSuccess ? SGR_OK : SGR_ERR_CUDA;
}

sgr_status_t sgr_combine_summaries(sgr_op_t op, const float *pairs, int64_t rank, const void *init,
                                   int64_t init_bs, void *out, int64_t out_bs, int64_t B, int64_t D,
                                   sgr_dtype_t dtype, cudaStream_t stream) {
    if (dtype != SGR_F32 && dtype != SGR_BF16) return SGR_ERR_INVALID_ARG;
    if (op != SGR_OP_MINGRU && op != SGR_OP_MINMAX) return SGR_ERR_INVALID_ARG;
    if (B < 0 || D < 0 || rank < 0 || init_bs < 0 || out_bs < 0) return SGR_ERR_INVALID_ARG;
    if (B == 0 || D == 0) return SGR_OK;
    if (!out || (rank > 0 && !pairs)) return SGR_ERR_INVALID_ARG;
    if (B > 1 && out_bs < D) return SGR_ERR_INVALID_ARG;
    const int esz = dtype == SGR_BF16 ? 2 : 4;
    int64_t tmp = 0;
    for (int64_t bs : {init_bs, out_bs})
        if (!mul_ok(B - 1, bs, &tmp) || !mul_ok(tmp + D, esz, &tmp)) return SGR_ERR_UNSUPPORTED;
    if (!mul_ok(rank, B, &tmp) || !mul_ok(tmp, D, &tmp) || !mul_ok(tmp, 8, &tmp)) return SGR_ERR_UNSUPPORTED;
    const size_t ob = rows_span(B, D, out_bs, esz);
    if (overlaps(out, ob, pairs, size_t(tmp))) return SGR_ERR_INVALID_ARG;
    const bool in_place = init == out && init_bs == out_bs;
    if (init && !in_place && overlaps(out, ob, init, rows_span(B, D, init_bs, esz)))
        return SGR_ERR_INVALID_ARG;
    const int64_t BD = B * D;
    const unsigned grid = unsigned(std::min<int64_t>((BD + 255) / 256, int64_t(kAssumedSMs) * 16));
    const float2 *pp = reinterpret_cast<const float2 *>(pairs);
    if (op == SGR_OP_MINGRU) {
        if (dtype == SGR_F32)
            combine_summaries_kernel<MinGRUOp, float><<<grid, 256, 0, stream>>>(
                pp, rank, static_cast<const float *>(init), init_bs, static_cast<float *>(out), out_bs, B, D);
        else
            combine_summaries_kernel<MinGRUOp, __nv_bfloat16><<<grid, 256, 0, stream>>>(
                pp, rank, static_cast<const __nv_bfloat16 *>(init), init_bs,
                static_cast<__nv_bfloat16 *>(out), out_bs, B, D);
    } else {
        if (dtype == SGR_F32)
            combine_summaries_kernel<MinMaxOp, float><<<grid, 256, 0, stream>>>(
                pp, rank, static_cast<const float *>(init), init_bs, static_cast<float *>(out), out_bs, B, D);
        else
            combine_summaries_kernel<MinMaxOp, __nv_bfloat16><<<grid, 256, 0, stream>>>(
                pp, rank, static_cast<const __nv_bfloat16 *>(init), init_bs,
                static_cast<__nv_bfloat16 *>(out), out_bs, B, D);
    }
    return cudaGetLastError() == cudaSuccess ? SGR_OK : SGR_ERR_CUDA;
}

size_t sgr_backward_workspace_size(sgr_op_t op, int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype) {
    if (op != SGR_OP_MINGRU && op != SGR_OP_MINMAX) return 0;
    if (dtype != SGR_F32 && dtype != SGR_BF16) return 0;
    if (B <= 0 || T <= 0 || D <= 0) return 0;
    // the aligned and unaligned plans, plain and decayed (shorter tiles)
    size_t need = 0;
    for (int v = 0; v < 4; ++v)
        need = std::max(need, make_bwd_plan(B, T, D, dtype, (v & 1) == 0, v >= 2).ws_bytes);
    return need;
}

size_t sgr_workspace_size(sgr_op_t op, int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype) {
    if (op != SGR_OP_MINGRU && op != SGR_OP_MINMAX && op != SGR_OP_MINGRU_LOG) return 0;
    if (dtype != SGR_F32 && dtype != SGR_BF16) return 0;
    if (B <= 0 || T <= 0 || D <= 0) return 0;
    if (op == SGR_OP_MINGRU_LOG)
        return std::max(make_plan(B, T, D, dtype, true, false, false, false, true).ws_bytes,
                        make_plan(B, T, D, dtype, false, false, false, false, true).ws_bytes);
    // the vector and the scalar variant may cut T differently, and the
    // time-decayed minGRU may take another kernel: cover them all
    size_t need = 0;
    for (int v = 0; v < (op == SGR_OP_MINGRU ? 4 : 2); ++v)
        need = std::max(need, make_plan(B, T, D, dtype, (v & 1) == 0, false, op == SGR_OP_MINMAX, v >= 2).ws_bytes);
    return need;
}

sgr_status_t sgr_workspace_init(void *workspace, size_t ws_bytes, cudaStream_t stream) {
    if (ws_bytes == 0) return SGR_OK;
    if (!workspace) return SGR_ERR_INVALID_ARG;
    return cudaMemsetAsync(workspace, 0, ws_bytes, stream) == cudaSuccess ? SGR_OK : SGR_ERR_CUDA;
}

sgr_status_t sgr_workspace_status(void *workspace, size_t ws_bytes, int clear, cudaStream_t stream) {
    if (!workspace || ws_bytes < sizeof(uint32_t)) return SGR_ERR_INVALID_ARG;
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return SGR_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return SGR_ERR_CUDA;
    if (clear) {
        if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), stream) != cudaSuccess) return SGR_ERR_CUDA;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return SGR_ERR_CUDA;
    }
    return (word & sgr::kTimeoutBit) ? SGR_ERR_TIMEOUT : SGR_OK;
}

const char *sgr_status_string(sgr_status_t s) {
    switch (s) {
        case SGR_OK: return "ok";
        case SGR_ERR_INVALID_ARG: return "invalid argument";
        case SGR_ERR_UNSUPPORTED: return "unsupported size";
        case SGR_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case SGR_ERR_CUDA: return "CUDA error";
        case SGR_ERR_TIMEOUT: return "timed out waiting for an earlier chunk's state";
    }
    return "unknown status";
}

const char *sgr_version(void) { return "scan_gated_rnns_b200 0.1.0 sm_100a"; }

namespace {
void fill_plan(const Plan &p, sgr_plan_t *plan) {
    plan->vector_path = p.vec ? 1 : 0;
    plan->kernel = p.kind;
    plan->channels_per_thread = p.V;
    plan->channel_lanes = p.cg;
    plan->rows_per_thread = p.r;
    plan->warps = p.warps;
    const bool seq = seq_kind(p.kind);
    plan->threads = (seq ? plan->warps : plan->warps + 1) * 32;
    plan->stages = p.stages;
    plan->tile_rows = p.TR;
    plan->tile_channels = p.TC;
    plan->n_channel_tiles = p.n_dt;
    plan->n_chains = p.n_chains;
    plan->n_chunks = p.n_chunks;
    plan->n_tiles = p.n_tiles;
    plan->smem_bytes = p.smem;
    plan->workspace_bytes = p.ws_bytes;
    plan->off_words = p.off_words;
    if (p.n_chains > 0 && p.n_dt > 0 && p.n_chains < (int64_t(1) << 31)) {
        const FastDiv a = make_fastdiv(uint32_t(p.n_chains)), b = make_fastdiv(uint32_t(p.n_dt));
        plan->div_chains_m = a.m; plan->div_chains_s = a.s;
        plan->div_dt_m = b.m; plan->div_dt_s = b.s;
    } else {
        plan->div_chains_m = plan->div_chains_s = plan->div_dt_m = plan->div_dt_s = 0;
    }
}
}  // namespace

sgr_status_t sgr_scan_plan(sgr_op_t op, int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype,
                           int aligned, sgr_plan_t *plan) {
    if (op != SGR_OP_MINGRU && op != SGR_OP_MINMAX && op != SGR_OP_MINGRU_LOG) return SGR_ERR_INVALID_ARG;
    if (dtype != SGR_F32 && dtype != SGR_BF16) return SGR_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || D < 0 || !plan) return SGR_ERR_INVALID_ARG;
    fill_plan(make_plan(B, T, D, dtype, aligned != 0, false, op == SGR_OP_MINMAX, false, op == SGR_OP_MINGRU_LOG),
              plan);
    return SGR_OK;
}

sgr_status_t sgr_scan_plan_decay(int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype, int aligned,
                                 sgr_plan_t *plan) {
    if (dtype != SGR_F32 && dtype != SGR_BF16) return SGR_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || D < 0 || !plan) return SGR_ERR_INVALID_ARG;
    fill_plan(make_plan(B, T, D, dtype, aligned != 0, false, false, true), plan);
    return SGR_OK;
}

int sgr_backward_kernel(sgr_op_t op, int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype, int aligned) {
    if (op != SGR_OP_MINGRU && op != SGR_OP_MINMAX) return 0;
    if (dtype != SGR_F32 && dtype != SGR_BF16) return 0;
    if (B < 0 || T < 0 || D < 0) return 0;
    if (seq_backward_planned(B, T, D, dtype == SGR_BF16 ? 2 : 4, aligned != 0)) return KIND_SEQUENTIAL;
    return make_bwd_plan(B, T, D, dtype, aligned != 0).kind;
}

sgr_status_t sgr_set_wait_limit(uint32_t polls) {
    g_spin_limit.store(polls == 0 ? sgr::kSpinLimit : polls);
    return SGR_OK;
}

sgr_status_t sgr_set_drop_publish(int64_t tile) {
    if (tile < -1) return SGR_ERR_INVALID_ARG;
    g_drop_tile.store(tile);
    return SGR_OK;
}

sgr_status_t sgr_set_kernel_override(int kernel) {
    if (kernel < KIND_AUTO || kernel > KIND_SEQUENTIAL_QUAD) return SGR_ERR_INVALID_ARG;
    g_override_kind.store(kernel);
    return SGR_OK;
}

sgr_status_t sgr_set_tile_override(int channel_lanes, int rows_per_thread) {
    if (!(channel_lanes == 0 || channel_lanes == 8 || channel_lanes == 32)) return SGR_ERR_INVALID_ARG;
    if (!(rows_per_thread == 0 || rows_per_thread == 1 || rows_per_thread == 2 ||
          rows_per_thread == 4 || rows_per_thread == 8))
        return SGR_ERR_INVALID_ARG;
    g_override_cg.store(channel_lanes);
    g_override_r.store(rows_per_thread);
    return SGR_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// mingru_scan without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// scan: an inference runtime's plugin whose enqueue step must not call the
// allocator (allocation can block or fail in the middle of a run), a process
// with a fixed, pre-planned device-memory budget, or code that runs while its
// stream is being captured and must not make allocation calls there.  For
// them this entry point takes its scratch (the chunk hand-off words and the
// status word) from a fixed array that lives in the library itself.
//
// The array is kNoAllocScratchBytes (16 MiB) of device memory, held by every
// GPU that loads the library until the process exits.  The first call on a
// device looks up the array's device address (cudaGetSymbolAddress, with that
// device current) and zero-fills it on the caller's stream; that first call
// should therefore come before any stream capture.  All calls on a device
// share the one array and it keeps the last call's contents; every launch tags
// its hand-off words with a fresh epoch, so those need no clearing between
// calls, but calls whose kernels can overlap on the GPU (e.g. on two streams
// without an ordering between them) race on the array and must not be made.
// The array's status word is the library's own: each call clears it on the
// stream before its launch, and no entry point reads it back, so for this
// entry point a chunk that gave up waiting shows only as NaN outputs.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64] = {};

}  // namespace

extern "C" sgr_status_t mingru_scan_noalloc(const void *k, const void *hx, const void *h0,
                                            int64_t h0_batch_stride, void *h, int64_t B,
                                            int64_t T, int64_t D, sgr_dtype_t dtype,
                                            cudaStream_t stream) {
    if (dtype != SGR_F32 && dtype != SGR_BF16) return SGR_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || D < 0 || h0_batch_stride < 0) return SGR_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || D == 0) return SGR_OK;
    // scratch this shape needs, for whichever kernel variant the call takes
    const size_t need = sgr_workspace_size(SGR_OP_MINGRU, B, T, D, dtype);
    if (need > kNoAllocScratchBytes) return SGR_ERR_WORKSPACE;
    if (!k || !hx || !h) return SGR_ERR_INVALID_ARG;
    void *ws = nullptr;
    if (need > 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SGR_ERR_CUDA;
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (g_noalloc_ptr[dev] == nullptr) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
                return SGR_ERR_CUDA;
            if (cudaMemsetAsync(p, 0, kNoAllocScratchBytes, stream) != cudaSuccess) return SGR_ERR_CUDA;
            g_noalloc_ptr[dev] = p;
        }
        ws = g_noalloc_ptr[dev];
        // a bit left by an earlier call's timed-out wait must not linger
        if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), stream) != cudaSuccess) return SGR_ERR_CUDA;
    }
    return mingru_scan(k, hx, h0, h0_batch_stride, h, B, T, D, dtype, ws,
                       ws ? kNoAllocScratchBytes : 0, stream);
}
