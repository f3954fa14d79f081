// scan_sequential.cuh -- channel-sequential scan for wide batches, sm_100a.
//
// When a scan has enough channels (B x D) to give every SM several warps, the
// time axis needs no splitting at all: each warp takes a group of channels of
// one batch row and walks t = 0 .. T-1 in order, applying each step's map to
// the state it holds in registers,
//   minGRU (page "Mingru Pytorch", log-space minGRU): h <- a_t h + b_t,
//       a_t = 1 - z_t = sigmoid(-k_t), b_t = z_t g(hx_t);
//   MinMax neuron (page "MinMax Recurrent Neural Cascades", The model, item 3):
//       x <- max(min(x, r_t), s_t).
// This is the chunked scan with one chunk per channel: there is no fold of a
// chunk into a summary pair, no carry between blocks and no replay, so per
// element the work is the activations and one step.  The parallel (chunked)
// kernels in scan_engine.cuh remain for shapes with fewer channels, where the
// time axis has to be cut to fill the GPU.
//
// Layout per warp (the one-warp kernel; the two-warp kernels below split
// each slot's rows between a pair of warps, and the bf16 form with 64-channel
// groups gives each lane two channels): a channel group of 32 channels (a
// 128-byte fp32 or 64-byte bf16 row segment per operand), lane l owning
// channel l of the group.  The
// warp streams its rows through a ring of S slots of
// RB rows in shared memory, both operands of a slot loaded by the tensor
// memory accelerator (one box of CW channels x RB rows per operand, completion
// counted on the slot's mbarrier; no multicast); lane 0 refills a slot as soon
// as the warp has copied it into registers.  Outputs go through two staging
// buffers of RB rows and leave by tensor-memory-accelerator stores (a bulk
// group per slot), so no thread computes an output address.  Every warp is
// independent: no block-wide barrier after set-up.  Rows past T and channels
// past D are zero-filled on load and clipped on store.
#pragma once

#include "scan_backward.cuh"
#include "scan_engine.cuh"

namespace sgr {

constexpr int kSeqRows = 16;          // rows per slot
constexpr int kSeqOutBufs = 2;

// one channel per lane: a warp's channel group is 32 channels, a 128-byte
// (fp32) or 64-byte (bf16) row segment per operand.  (Two bf16 channels per
// lane halve the warps a batch provides; the warps' latency, not their issue
// rate, bounds this kernel, and 32-channel groups measured 13-40% faster.)
template <typename IO> constexpr int seq_row_bytes() { return 32 * int(sizeof(IO)); }

// Time decay through the copy engine: each slot carries its 16 rows' gaps
// (a 64-byte box of the (B, T) gap array) in a 128-byte area after its
// operand boxes, so they land with the slot on its mbarrier.
constexpr uint32_t kSeqGapBytes = 128;

// bytes of one warp's shared memory with S load slots of rows of `row_bytes`
// (gap: the per-slot gap area, 0 or kSeqGapBytes)
__host__ __device__ constexpr size_t seq_warp_bytes(int S, int row_bytes, size_t gap = 0) {
    return (size_t(S) * (2 * kSeqRows * row_bytes + gap) + size_t(kSeqOutBufs) * kSeqRows * row_bytes +
            size_t(S) * 8 + 127) / 128 * 128;
}

// a lane's element of one row in shared memory, widened to / narrowed from fp32
template <typename IO> struct LaneRow;
template <> struct LaneRow<float> {
    static __device__ __forceinline__ float load(uint32_t a) {
        uint32_t v;
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
        return __uint_as_float(v);
    }
    static __device__ __forceinline__ void store(uint32_t a, float x) {
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(__float_as_uint(x)) : "memory");
    }
};
template <> struct LaneRow<__nv_bfloat16> {
    static __device__ __forceinline__ float load(uint32_t a) {
        uint16_t v;
        asm volatile("ld.shared.b16 %0, [%1];" : "=h"(v) : "r"(a) : "memory");
        return __uint_as_float(uint32_t(v) << 16);
    }
    static __device__ __forceinline__ void store(uint32_t a, float x) {
        __nv_bfloat16 h = __float2bfloat16_rn(x);
        asm volatile("st.shared.b16 [%0], %1;" ::"r"(a), "h"(*reinterpret_cast<uint16_t *>(&h)) : "memory");
    }
};

// shared -> global tensor store of one box (a bulk group per call)
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, uint32_t src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most N of this thread's bulk groups still reading shared memory
template <int N> __device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

struct SeqParams {
    ScanParams s;        // operands, sizes, initial state, status word (may be null), decay
    int64_t n_groups;    // channel groups per batch row
    int64_t n_warps;     // B * n_groups
    int slots;           // load ring depth S
};

// The step pairs of two rows: bf16 I/O takes the shared-reciprocal form
// (one MUFU operation fewer per element; these kernels keep the MUFU pipe
// busy), fp32 I/O the form with relative-accurate gates for either sign.
template <class Op, typename IO>
__device__ __forceinline__ void seq_rows(float k0, float hx0, float k1, float hx1, float2 &a, float2 &b) {
    if constexpr (sizeof(IO) == 2 && Op::kLeanRows) Op::element_rows_lean(k0, hx0, k1, hx1, a, b);
    else Op::element_rows(k0, hx0, k1, hx1, a, b);
}

// Time decay in the channel-sequential kernels: the gaps u_t are per (batch
// row, row), shared by a warp's channels.  A warp's 16 rows of a slot have
// their gaps spread across the lanes, lane l holding row y0 + (l % 16)'s
// (0 past T: gamma = 1) -- read from the slot's gap box where the copy engine
// brings it (seq_smem_gap), else loaded two slots ahead (seq_slot_gap) so
// that no step waits for them; each row's gap is then taken from its lane by
// one shuffle.
__device__ __forceinline__ float seq_slot_gap(const ScanParams &p, int64_t b, int64_t y0, int lane) {
    const int64_t t = y0 + (lane & (kSeqRows - 1));
    return (y0 >= 0 && t < p.T) ? decay_u(p, b, t) : 0.f;
}
// the decay gates of two elements with their exponents in one packed
// multiply: (2^(l.x u.x), 2^(l.y u.y)), each product as decay_gamma's
__device__ __forceinline__ float2 decay_gamma2(float2 l, float2 u) {
    const float2 e = __fmul2_rn(l, u);
    return make_float2(fast_exp2(e.x), fast_exp2(e.y));
}
// the same gap from a slot's gap area (rows past T were zero-filled: gamma = 1)
__device__ __forceinline__ float seq_smem_gap(const ScanParams &p, uint32_t gaps, int lane) {
    float g;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(g) : "r"(gaps + 4u * uint32_t(lane & (kSeqRows - 1))) : "memory");
    return p.decay_log1p ? log1pf(g) : g;
}

// Block: WB independent warps; warp (blockIdx.x WB + w) scans channel group
// (b, grp) of the batch.  Dynamic shared memory: WB x seq_warp_bytes(S).
//
// SPLIT = 1: a warp's group is 32 channels, lane l owns channel l and walks
// every row.  SPLIT = 2: a warp's group is 16 channels and each slot's rows
// are split between the two half-warps, which doubles the warps a batch
// provides (the kernel is bound by the latency each warp exposes, so twice
// the warps hide it better) at the price of a fold and a hand-off per slot:
// lane (c, part) = (lane % 16, lane / 16) owns channel c of rows
// [8 part, 8 part + 8) of every slot.  Both halves fold their 8 step maps
// into one pair; the lower half applies its pair to the slot's incoming
// state, hands the result (the state after row 7) to the upper half with one
// shuffle, the upper half applies its own pair to it and hands the slot's
// final state back; then every lane replays its 8 rows from its incoming
// state and stores them.  This is the chunked scan with two chunks per slot
// (page "MinMax Recurrent Neural Cascades", Key properties: the pairs
// compose associatively).  The two halves read rows 256 (bf16) or 512
// (fp32) bytes apart, a 2-way shared-memory bank conflict per load.
template <class Op, typename IO, int WB, int SPLIT = 1, bool DT = false>
__global__ void __launch_bounds__(WB * 32)
scan_sequential_kernel(const SeqParams q, const __grid_constant__ CUtensorMap map0,
                       const __grid_constant__ CUtensorMap map1, const __grid_constant__ CUtensorMap map_out,
                       const __grid_constant__ CUtensorMap map_gap) {
    static_assert(SPLIT == 1 || SPLIT == 2, "one or two row groups per slot");
    static_assert(!DT || Op::kDecay, "gaps through the copy engine need a decay operator");
    static_assert(!Op::kLogSpace, "the channel-sequential kernels carry linear states");
    constexpr uint32_t kGap = DT ? kSeqGapBytes : 0;
    using LR = LaneRow<IO>;
    constexpr int CW = 32 / SPLIT;                                   // channels of a warp's group
    constexpr int LROWS = kSeqRows / SPLIT;                          // rows of a slot per lane
    constexpr int kRowBytes = CW * int(sizeof(IO));
    constexpr uint32_t kOpBytes = kSeqRows * kRowBytes;             // one operand of a slot
    static_assert(LROWS % 2 == 0, "rows are taken in pairs");
    const ScanParams &p = q.s;
    extern __shared__ __align__(128) unsigned char smem[];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t gw = int64_t(blockIdx.x) * WB + warp;
    if (gw >= q.n_warps) return;                                     // no block barrier below
    const int S = q.slots;
    const int64_t b = gw / q.n_groups;
    const int64_t grp = gw - b * q.n_groups;
    const int x0 = int(grp) * CW;                                    // first channel of the group
    const int ch = lane % CW;                                        // the lane's channel in the group
    const int part = lane / CW;                                      // the lane's rows of a slot
    const int64_t d = int64_t(x0) + ch;                              // the lane's channel

    constexpr uint32_t kSlot = 2 * kOpBytes + kGap;                 // [k rows | hx rows | gaps]
    const uint32_t base = smem_addr(smem) + uint32_t(warp * seq_warp_bytes(S, kRowBytes, kGap));
    const uint32_t ring = base;                                      // S slots
    const uint32_t outb = base + uint32_t(S) * kSlot;                // 2 staging buffers
    const uint32_t bars = outb + kSeqOutBufs * kOpBytes;             // S mbarriers
    const uint32_t lane_off = uint32_t(part * LROWS * kRowBytes + ch * int(sizeof(IO)));

    const int n_slots = int((p.T + kSeqRows - 1) / kSeqRows);       // T < 2^31 (host check)
    auto issue = [&](int i, int s) {                                 // lane 0: rows of slot i into ring slot s
        const uint32_t dst = ring + uint32_t(s) * kSlot;
        const uint32_t bar = bars + 8u * uint32_t(s);
        mbar_expect_tx(bar, 2 * kOpBytes + (DT ? kSeqRows * 4 : 0));
        tma_load_3d(dst, &map0, x0, i * kSeqRows, int(b), bar);
        tma_load_3d(dst + kOpBytes, &map1, x0, i * kSeqRows, int(b), bar);
        if constexpr (DT) tma_load_2d(dst + 2 * kOpBytes, &map_gap, i * kSeqRows, int(b), bar);
    };
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bars + 8u * s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int s = 0; s < S && s < n_slots; ++s) issue(s, s);
    }
    __syncwarp();

    float h = load_init<IO>(p, b, d, Op::default_init());           // state entering the slot
    [[maybe_unused]] float lam2 = 0.f, gcur = 0.f;
    [[maybe_unused]] float gnext = 0.f;
    if constexpr (Op::kDecay) {
        lam2 = decay_lam2(p, d);
        if constexpr (!DT) {
            gcur = seq_slot_gap(p, b, 0, lane);
            gnext = seq_slot_gap(p, b, kSeqRows, lane);
        }
    }

    uint32_t wait_limit = kMbarLimit;
    bool bad = false;
    int s = 0;                 // ring slot of slot i
    uint32_t phase = 0;        // parity of that slot's current use
    for (int i = 0; i < n_slots; ++i) {
        [[maybe_unused]] float gnext2 = 0.f;
        if constexpr (Op::kDecay && !DT) gnext2 = seq_slot_gap(p, b, int64_t(i + 2) * kSeqRows, lane);
        if (!mbar_wait(bars + 8u * uint32_t(s), phase, wait_limit)) {
            // a copy that never lands: record it, make every later output NaN
            // and stop waiting at length (the kernel still ends)
            wait_limit = 1;
            if (!bad && lane == 0 && p.status) atomicOr(p.status, kTimeoutBit);
            bad = true;
        }
        const uint32_t src = ring + uint32_t(s) * kSlot + lane_off;
        float x0r[LROWS], x1r[LROWS];
#pragma unroll
        for (int r = 0; r < LROWS; ++r) {
            x0r[r] = LR::load(src + r * kRowBytes);
            x1r[r] = LR::load(src + kOpBytes + r * kRowBytes);
        }
        if constexpr (DT) gcur = seq_smem_gap(p, ring + uint32_t(s) * kSlot + 2 * kOpBytes, lane);
        // staging buffer i % 2 is free once the store issued two slots ago
        // has read it (the warp synchronises just below)
        if (lane == 0) bulk_wait_read<kSeqOutBufs - 1>();
        __syncwarp();                                                // the slot is in registers
        if (lane == 0 && !bad && i + S < n_slots) {
            fence_proxy_async();
            issue(i + S, s);
        }
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }
        const uint32_t obuf = outb + uint32_t(i & (kSeqOutBufs - 1)) * kOpBytes;
        const uint32_t dst = obuf + lane_off;
        if (__any_sync(0xffffffffu, bad)) {
            // a copy of this or an earlier slot never landed: NaN outputs
            bad = true;
#pragma unroll
            for (int r = 0; r < LROWS; ++r) LR::store(dst + r * kRowBytes, __int_as_float(0x7fffffff));
        } else if constexpr (SPLIT == 1) {
            // the step maps of two rows at a time (independent of the
            // state), then the two steps
#pragma unroll
            for (int r = 0; r < LROWS; r += 2) {
                float2 a, c;
                seq_rows<Op, IO>(x0r[r], x1r[r], x0r[r + 1], x1r[r + 1], a, c);
                if constexpr (Op::kDecay) {
                    a = __fmul2_rn(a, decay_gamma2(make_float2(lam2, lam2),
                                                   make_float2(__shfl_sync(0xffffffffu, gcur, r),
                                                               __shfl_sync(0xffffffffu, gcur, r + 1))));
                }
                h = Op::step(a.x, c.x, h);
                LR::store(dst + r * kRowBytes, h);
                h = Op::step(a.y, c.y, h);
                LR::store(dst + (r + 1) * kRowBytes, h);
            }
        } else {
            // the lane's step maps, their fold into one pair, the hand-off
            // between the two halves, then the replay from the lane's state
            float am[LROWS], cm[LROWS];
#pragma unroll
            for (int r = 0; r < LROWS; r += 2) {
                float2 a, c;
                seq_rows<Op, IO>(x0r[r], x1r[r], x0r[r + 1], x1r[r + 1], a, c);
                if constexpr (Op::kDecay) {
                    a = __fmul2_rn(a, decay_gamma2(make_float2(lam2, lam2),
                                                   make_float2(__shfl_sync(0xffffffffu, gcur, part * LROWS + r),
                                                               __shfl_sync(0xffffffffu, gcur, part * LROWS + r + 1))));
                }
                am[r] = a.x; cm[r] = c.x;
                am[r + 1] = a.y; cm[r + 1] = c.y;
            }
            float2 P = make_float2(am[0], cm[0]);
#pragma unroll
            for (int r = 1; r < LROWS; ++r) P = Op::combine(P, make_float2(am[r], cm[r]));
            const float lo_out = Op::apply(P, h);                        // lower half: state after row LROWS-1
            const float from_lo = __shfl_xor_sync(0xffffffffu, lo_out, 16);
            const float hin = part ? from_lo : h;                        // the lane's incoming state
            const float out = Op::apply(P, hin);                         // upper half: the slot's final state
            const float from_hi = __shfl_xor_sync(0xffffffffu, out, 16);
            h = part ? out : from_hi;
            float y = hin;
#pragma unroll
            for (int r = 0; r < LROWS; ++r) {
                y = Op::step(am[r], cm[r], y);
                LR::store(dst + r * kRowBytes, y);
            }
        }
        fence_proxy_async();                                         // outputs visible to the store
        __syncwarp();
        if (lane == 0) {
            tma_store_3d(&map_out, obuf, x0, i * kSeqRows, int(b));
            bulk_commit();
        }
        if constexpr (Op::kDecay && !DT) {
            gcur = gnext;
            gnext = gnext2;
        }
    }
    if (lane == 0) bulk_wait_all();
}

// Two warps per channel group, each slot's rows split between them (wide bf16
// batches whose 32-channel groups alone leave each SM short of warps): the
// block's warps w = 0, 1 scan the same 32 channels of one batch row (lane =
// channel, 64- or 128-byte rows, no bank conflicts), warp w taking rows
// [32 i + 16 w, 32 i + 16 w + 16) of slot i through its own ring of 16-row
// boxes.  Each warp folds its 16 step maps into one pair -- rows r and r + 8
// as two chains, one fp32x2 operation advancing both, the running composites
// kept -- and puts it in shared memory (double-buffered by slot parity); after one named barrier per
// slot both warps read the other's pair and compose the slot's chain
// themselves -- h_mid = P0(h), h_end = P1(h_mid) -- so no second hand-off is
// needed: warp 0 takes h, warp 1 h_mid as its incoming state, and both carry
// h_end into the next slot.  A row's output is then its chain's running
// composite applied to the chain's incoming state, one independent fp32x2
// operation for two rows (no replay chain).  A warp whose copy never landed publishes a NaN
// pair, so both warps' later outputs turn NaN.  One staging buffer per warp
// (its previous store has long finished reading it by the time the next
// slot's outputs are written), which leaves the shared memory to the load
// ring.  Dynamic shared memory: 2 x seq_pair_warp_bytes(S) + the pair buffers.
constexpr int kPairWarps = 2;
// rows: a warp's rows of a slot (16; 8 in the four-warp blocks)
__host__ __device__ constexpr size_t seq_pair_warp_bytes(int S, int row_bytes, size_t gap = 0, int rows = kSeqRows) {
    return (size_t(S) * (2 * rows * row_bytes + gap) + size_t(rows) * row_bytes + size_t(S) * 8 + 127) / 128 * 128;
}
__host__ __device__ constexpr size_t seq_pair_block_bytes(int S, int row_bytes, size_t gap = 0) {
    return kPairWarps * seq_pair_warp_bytes(S, row_bytes, gap) + size_t(2) * kPairWarps * 32 * sizeof(float2);
}

template <class Op, typename IO, bool DT = false>
__global__ void __launch_bounds__(kPairWarps * 32)
scan_sequential_pair_kernel(const SeqParams q, const __grid_constant__ CUtensorMap map0,
                            const __grid_constant__ CUtensorMap map1, const __grid_constant__ CUtensorMap map_out,
                            const __grid_constant__ CUtensorMap map_gap) {
    static_assert(!DT || Op::kDecay, "gaps through the copy engine need a decay operator");
    static_assert(!Op::kLogSpace, "the channel-sequential kernels carry linear states");
    constexpr uint32_t kGap = DT ? kSeqGapBytes : 0;
    using LR = LaneRow<IO>;
    constexpr int CW = 32;
    constexpr int kRowBytes = CW * int(sizeof(IO));
    constexpr uint32_t kOpBytes = kSeqRows * kRowBytes;             // one operand of a warp's 16 rows
    constexpr int kSlotRows = kPairWarps * kSeqRows;                // rows of a slot (both warps)
    const ScanParams &p = q.s;
    extern __shared__ __align__(128) unsigned char smem[];

    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int64_t gw = blockIdx.x;                                   // one channel group per block
    if (gw >= q.n_warps) return;                                     // whole block: no barrier is left waiting
    const int S = q.slots;
    const int64_t b = gw / q.n_groups;
    const int64_t grp = gw - b * q.n_groups;
    const int x0 = int(grp) * CW;
    const int64_t d = int64_t(x0) + lane;

    constexpr uint32_t kSlot = 2 * kOpBytes + kGap;                 // [k rows | hx rows | gaps]
    const uint32_t base = smem_addr(smem) + uint32_t(w * seq_pair_warp_bytes(S, kRowBytes, kGap));
    const uint32_t ring = base;
    const uint32_t outb = base + uint32_t(S) * kSlot;               // one staging buffer
    const uint32_t bars = outb + kOpBytes;
    float2 *xpair = reinterpret_cast<float2 *>(smem + kPairWarps * seq_pair_warp_bytes(S, kRowBytes, kGap));  // [2][2][32]

    const int n_slots = int((p.T + kSlotRows - 1) / kSlotRows);     // T < 2^31 (host check)
    auto issue = [&](int i, int s) {
        const uint32_t dst = ring + uint32_t(s) * kSlot;
        const uint32_t bar = bars + 8u * uint32_t(s);
        const int y = i * kSlotRows + w * kSeqRows;
        mbar_expect_tx(bar, 2 * kOpBytes + (DT ? kSeqRows * 4 : 0));
        tma_load_3d(dst, &map0, x0, y, int(b), bar);
        tma_load_3d(dst + kOpBytes, &map1, x0, y, int(b), bar);
        if constexpr (DT) tma_load_2d(dst + 2 * kOpBytes, &map_gap, y, int(b), bar);
    };
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bars + 8u * s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int s = 0; s < S && s < n_slots; ++s) issue(s, s);
    }
    __syncwarp();

    float h = load_init<IO>(p, b, d, Op::default_init());           // state entering the slot
    [[maybe_unused]] float lam2 = 0.f, gcur = 0.f;
    [[maybe_unused]] float gnext = 0.f;
    if constexpr (Op::kDecay) {
        lam2 = decay_lam2(p, d);
        if constexpr (!DT) {
            gcur = seq_slot_gap(p, b, w * kSeqRows, lane);
            gnext = seq_slot_gap(p, b, kSlotRows + w * kSeqRows, lane);
        }
    }

    uint32_t wait_limit = kMbarLimit;
    bool bad = false;
    int s = 0;
    uint32_t phase = 0;
    for (int i = 0; i < n_slots; ++i) {
        [[maybe_unused]] float gnext2 = 0.f;
        if constexpr (Op::kDecay && !DT)
            gnext2 = seq_slot_gap(p, b, int64_t(i + 2) * kSlotRows + w * kSeqRows, lane);
        if (!mbar_wait(bars + 8u * uint32_t(s), phase, wait_limit)) {
            wait_limit = 1;
            if (!bad && lane == 0 && p.status) atomicOr(p.status, kTimeoutBit);
            bad = true;
        }
        const uint32_t src = ring + uint32_t(s) * kSlot + uint32_t(lane) * uint32_t(sizeof(IO));
        float x0r[kSeqRows], x1r[kSeqRows];
#pragma unroll
        for (int r = 0; r < kSeqRows; ++r) {
            x0r[r] = LR::load(src + r * kRowBytes);
            x1r[r] = LR::load(src + kOpBytes + r * kRowBytes);
        }
        if constexpr (DT) gcur = seq_smem_gap(p, ring + uint32_t(s) * kSlot + 2 * kOpBytes, lane);
        __syncwarp();                                                // the slot is in registers
        if (lane == 0 && !bad && i + S < n_slots) {
            fence_proxy_async();
            issue(i + S, s);
        }
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }
        bad = __any_sync(0xffffffffu, bad);
        // rows r and r + 8 as two chains, each fp32x2 operation spanning
        // both: the step maps of the pair, then the running composites from
        // the start of each chain (PA, PB: the pair mapping the chain's
        // incoming state to row r's, resp. row r + 8's, output)
        constexpr int H = kSeqRows / 2;
        float2 PA[H], PB[H];
        float2 A = make_float2(Op::identity().x, Op::identity().x);
        float2 Bc = make_float2(Op::identity().y, Op::identity().y);
#pragma unroll
        for (int r = 0; r < H; ++r) {
            float2 a, c;
            seq_rows<Op, IO>(x0r[r], x1r[r], x0r[r + H], x1r[r + H], a, c);
            if constexpr (Op::kDecay) {
                a = __fmul2_rn(a, decay_gamma2(make_float2(lam2, lam2),
                                               make_float2(__shfl_sync(0xffffffffu, gcur, r),
                                                           __shfl_sync(0xffffffffu, gcur, r + H))));
            }
            Op::fold2(A, Bc, a, c);
            PA[r] = A;
            PB[r] = Bc;
        }
        // the warp's 16 rows: the first chain, then the second
        float2 P = Op::combine(make_float2(A.x, Bc.x), make_float2(A.y, Bc.y));
        if (bad) P = make_float2(__int_as_float(0x7fffffff), __int_as_float(0x7fffffff));
        float2 *xb = xpair + (i & 1) * kPairWarps * 32;
        xb[w * 32 + lane] = P;
        named_barrier_sync(1, kPairWarps * 32);                      // both warps' pairs of slot i written
        const float2 Q = xb[(1 - w) * 32 + lane];
        const float hmid = Op::apply(w ? Q : P, h);
        const float hend = Op::apply(w ? P : Q, hmid);
        const float hin = w ? hmid : h;                              // this warp's incoming state
        h = hend;
        // incoming states of the two chains: the warp's, and the state after row 7
        float2 hh = make_float2(hin, Op::apply(make_float2(A.x, Bc.x), hin));
        if (bad) hh = make_float2(__int_as_float(0x7fffffff), __int_as_float(0x7fffffff));   // NaN outputs
        if (lane == 0) bulk_wait_read<0>();                          // the last slot's store has read the buffer
        __syncwarp();
        const uint32_t obuf = outb;
        const uint32_t dst = obuf + uint32_t(lane) * uint32_t(sizeof(IO));
#pragma unroll
        for (int r = 0; r < H; ++r) {
            const float2 y = Op::step2(PA[r], PB[r], hh);           // rows r and r + 8, independent
            LR::store(dst + r * kRowBytes, y.x);
            LR::store(dst + (r + H) * kRowBytes, y.y);
        }
        fence_proxy_async();
        __syncwarp();
        const int y0 = i * kSlotRows + w * kSeqRows;
        if (lane == 0 && y0 < p.T) {                                  // no store starts past the tensor
            tma_store_3d(&map_out, obuf, x0, y0, int(b));
            bulk_commit();
        }
        if constexpr (Op::kDecay && !DT) {
            gcur = gnext;
            gnext = gnext2;
        }
    }
    if (lane == 0) bulk_wait_all();
}

// The two-warp kernel with two channels per lane (bf16 I/O): a block scans a
// group of 64 channels of one batch row, lane l owning channels 2l and
// 2l + 1, so each operand row of a warp is one 128-byte segment read as one
// 32-bit shared load per lane, and each output row is written as one packed
// bf16 pair.  Everything else follows scan_sequential_pair_kernel: with NW
// warps per block and RW = 32 / NW rows per warp, warp w takes rows
// [32 i + RW w, 32 i + RW w + RW) of slot i through its own ring, folds them
// -- here four chains per lane (two channels x rows r and r + RW / 2),
// advanced as two fp32x2 operations per row pair -- exchanges its two pairs
// with the other warps after one named barrier per slot (each warp composes
// the slot's NW pairs in row order from the slot's incoming state, keeping
// the state in front of its own rows), and writes each row as its chain's
// running composite applied to the chain's incoming state.  The channel pair
// doubles each warp's independent work while the batch provides half the
// warps; four warps per group (8 rows each) bring the warp count back to
// that of the 32-channel pairs.
constexpr int kPair2Channels = 64;
constexpr int kQuadWarps = 4;
__host__ __device__ constexpr size_t seq_pair2_block_bytes(int S, size_t gap = 0, int NW = kPairWarps) {
    return size_t(NW) * seq_pair_warp_bytes(S, kPair2Channels * 2, gap, 32 / NW) +
           size_t(2) * size_t(NW) * 32 * sizeof(float4);
}

// two bf16 channels of one row: (low, high) halves as fp32
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void sts_bf16x2(uint32_t a, float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(*reinterpret_cast<const uint32_t *>(&h)) : "memory");
}

template <class Op, bool DT = false, int NW = kPairWarps>
__global__ void __launch_bounds__(NW * 32)
scan_sequential_pair2_kernel(const SeqParams q, const __grid_constant__ CUtensorMap map0,
                             const __grid_constant__ CUtensorMap map1, const __grid_constant__ CUtensorMap map_out,
                             const __grid_constant__ CUtensorMap map_gap) {
    static_assert(!DT || Op::kDecay, "gaps through the copy engine need a decay operator");
    static_assert(!Op::kLogSpace, "the channel-sequential kernels carry linear states");
    static_assert(NW == kPairWarps || NW == kQuadWarps, "two or four warps per group");
    using IO = __nv_bfloat16;
    constexpr uint32_t kGap = DT ? kSeqGapBytes : 0;
    constexpr int CW = kPair2Channels;
    constexpr int RW = 32 / NW;                                     // a warp's rows of a slot
    constexpr int kRowBytes = CW * int(sizeof(IO));                 // 128
    constexpr uint32_t kOpBytes = RW * kRowBytes;                   // one operand of a warp's rows
    constexpr int kSlotRows = NW * RW;
    constexpr int H = RW / 2;
    const ScanParams &p = q.s;
    extern __shared__ __align__(128) unsigned char smem[];

    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int64_t gw = blockIdx.x;
    if (gw >= q.n_warps) return;
    const int S = q.slots;
    const int64_t b = gw / q.n_groups;
    const int64_t grp = gw - b * q.n_groups;
    const int x0 = int(grp) * CW;
    const int64_t d = int64_t(x0) + 2 * lane;                       // the lane's first channel

    // the slot's gap box is 16 rows (a warp of four-warp blocks uses 8 of them)
    constexpr uint32_t kSlot = 2 * kOpBytes + kGap;
    const uint32_t base = smem_addr(smem) + uint32_t(w * seq_pair_warp_bytes(S, kRowBytes, kGap, RW));
    const uint32_t ring = base;
    const uint32_t outb = base + uint32_t(S) * kSlot;
    const uint32_t bars = outb + kOpBytes;
    float4 *xpair = reinterpret_cast<float4 *>(smem + NW * seq_pair_warp_bytes(S, kRowBytes, kGap, RW));  // [2][NW][32]

    const int n_slots = int((p.T + kSlotRows - 1) / kSlotRows);
    auto issue = [&](int i, int s) {
        const uint32_t dst = ring + uint32_t(s) * kSlot;
        const uint32_t bar = bars + 8u * uint32_t(s);
        const int y = i * kSlotRows + w * RW;
        mbar_expect_tx(bar, 2 * kOpBytes + (DT ? kSeqRows * 4 : 0));
        tma_load_3d(dst, &map0, x0, y, int(b), bar);
        tma_load_3d(dst + kOpBytes, &map1, x0, y, int(b), bar);
        if constexpr (DT) tma_load_2d(dst + 2 * kOpBytes, &map_gap, y, int(b), bar);
    };
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bars + 8u * s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int s = 0; s < S && s < n_slots; ++s) issue(s, s);
    }
    __syncwarp();

    // states entering the slot (channels d, d + 1; past D: the default)
    float2 h = make_float2(load_init<IO>(p, b, d, Op::default_init()), load_init<IO>(p, b, d + 1, Op::default_init()));
    [[maybe_unused]] float2 lam2 = make_float2(0.f, 0.f);
    [[maybe_unused]] float gcur = 0.f, gnext = 0.f;
    if constexpr (Op::kDecay) {
        lam2 = make_float2(d < p.D ? decay_lam2(p, d) : 0.f, d + 1 < p.D ? decay_lam2(p, d + 1) : 0.f);
        if constexpr (!DT) {
            gcur = seq_slot_gap(p, b, w * RW, lane);
            gnext = seq_slot_gap(p, b, kSlotRows + w * RW, lane);
        }
    }

    uint32_t wait_limit = kMbarLimit;
    bool bad = false;
    int s = 0;
    uint32_t phase = 0;
    for (int i = 0; i < n_slots; ++i) {
        [[maybe_unused]] float gnext2 = 0.f;
        if constexpr (Op::kDecay && !DT)
            gnext2 = seq_slot_gap(p, b, int64_t(i + 2) * kSlotRows + w * RW, lane);
        if (!mbar_wait(bars + 8u * uint32_t(s), phase, wait_limit)) {
            wait_limit = 1;
            if (!bad && lane == 0 && p.status) atomicOr(p.status, kTimeoutBit);
            bad = true;
        }
        const uint32_t src = ring + uint32_t(s) * kSlot + uint32_t(lane) * 4u;
        uint32_t x0r[RW], x1r[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            x0r[r] = lds32(src + r * kRowBytes);
            x1r[r] = lds32(src + kOpBytes + r * kRowBytes);
        }
        if constexpr (DT) gcur = seq_smem_gap(p, ring + uint32_t(s) * kSlot + 2 * kOpBytes, lane);
        __syncwarp();                                                // the slot is in registers
        if (lane == 0 && !bad && i + S < n_slots) {
            fence_proxy_async();
            issue(i + S, s);
        }
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }
        bad = __any_sync(0xffffffffu, bad);
        // four chains: (channels d, d + 1) x (rows r, r + H); L = rows
        // [0, H), U = rows [H, RW), each an fp32x2 over the two channels
        float2 PAL[H], PBL[H], PAU[H], PBU[H];
        float2 AL = make_float2(Op::identity().x, Op::identity().x), BL = make_float2(Op::identity().y, Op::identity().y);
        float2 AU = AL, BU = BL;
#pragma unroll
        for (int r = 0; r < H; ++r) {
            const float2 kl = unpack_bf16x2(x0r[r]), hl = unpack_bf16x2(x1r[r]);
            const float2 ku = unpack_bf16x2(x0r[r + H]), hu = unpack_bf16x2(x1r[r + H]);
            float2 al, cl, au, cu;
            seq_rows<Op, IO>(kl.x, hl.x, kl.y, hl.y, al, cl);
            seq_rows<Op, IO>(ku.x, hu.x, ku.y, hu.y, au, cu);
            if constexpr (Op::kDecay) {
                const float ul = __shfl_sync(0xffffffffu, gcur, r), uu = __shfl_sync(0xffffffffu, gcur, r + H);
                al = __fmul2_rn(al, decay_gamma2(lam2, make_float2(ul, ul)));
                au = __fmul2_rn(au, decay_gamma2(lam2, make_float2(uu, uu)));
            }
            Op::fold2(AL, BL, al, cl);
            Op::fold2(AU, BU, au, cu);
            PAL[r] = AL;
            PBL[r] = BL;
            PAU[r] = AU;
            PBU[r] = BU;
        }
        // the warp's RW rows per channel: the first chain, then the second
        float4 P;
        {
            const float2 p0 = Op::combine(make_float2(AL.x, BL.x), make_float2(AU.x, BU.x));
            const float2 p1 = Op::combine(make_float2(AL.y, BL.y), make_float2(AU.y, BU.y));
            P = make_float4(p0.x, p0.y, p1.x, p1.y);
        }
        if (bad) P = make_float4(__int_as_float(0x7fffffff), __int_as_float(0x7fffffff), __int_as_float(0x7fffffff),
                                 __int_as_float(0x7fffffff));
        // the slot's pairs in row order (double-buffered by slot parity: a
        // buffer is written again two slots later, after every warp has read
        // it and passed the next slot's barrier)
        float4 *xb = xpair + (i & 1) * NW * 32;
        xb[w * 32 + lane] = P;
        named_barrier_sync(1, NW * 32);
        float2 hin = h;
#pragma unroll
        for (int j = 0; j < NW; ++j) {
            const float4 Pj = j == w ? P : xb[j * 32 + lane];
            if (j == w) hin = h;                                     // the state in front of this warp's rows
            h = make_float2(Op::apply(make_float2(Pj.x, Pj.y), h.x), Op::apply(make_float2(Pj.z, Pj.w), h.y));
        }
        // incoming states of the upper chains: after row H - 1 of each channel
        float2 hu = make_float2(Op::apply(make_float2(AL.x, BL.x), hin.x), Op::apply(make_float2(AL.y, BL.y), hin.y));
        float2 hl = hin;
        if (bad) {
            hl = make_float2(__int_as_float(0x7fffffff), __int_as_float(0x7fffffff));
            hu = hl;
        }
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        const uint32_t dst = outb + uint32_t(lane) * 4u;
#pragma unroll
        for (int r = 0; r < H; ++r) {
            const float2 yl = Op::step2(PAL[r], PBL[r], hl);
            const float2 yu = Op::step2(PAU[r], PBU[r], hu);
            sts_bf16x2(dst + r * kRowBytes, yl.x, yl.y);
            sts_bf16x2(dst + (r + H) * kRowBytes, yu.x, yu.y);
        }
        fence_proxy_async();
        __syncwarp();
        const int y0 = i * kSlotRows + w * RW;
        if (lane == 0 && y0 < p.T) {
            tma_store_3d(&map_out, outb, x0, y0, int(b));
            bulk_commit();
        }
        if constexpr (Op::kDecay && !DT) {
            gcur = gnext;
            gnext = gnext2;
        }
    }
    if (lane == 0) bulk_wait_all();
}

}  // namespace sgr

// ------------------------------------------------------- gradients
//
// The gradient of either scan walks the sequence backwards (scan_backward.cuh
// states the recurrence): with lam the gradient reaching out_t from the steps
// after t, delta = gy_t + lam, d in0_t = delta cP_t, d in1_t = delta cQ_t and
// lam <- A_t delta, where (A_t, cP_t, cQ_t) are the local partials of step t
// given the state before it (the forward output one row back, or the initial
// state at t = 0).  For wide batches each warp does this for its 32 channels
// from t = T - 1 down to 0 with lam in a register -- no reverse chunking, no
// look-back.  Slots are rows [j RB, j RB + RB) taken for j from the top down
// (the top one may run past T: those rows are skipped); per slot the copy
// engine brings four boxes -- k, hx (or r, s), gy, and the forward output
// shifted one row back (box starting at row j RB - 1; the row before t = 0
// is read as zero fill and replaced by the initial state) -- and two boxes of
// input gradients leave by tensor stores, which never start at a negative row.
namespace sgr {

constexpr int kSeqBwdIn = 4;        // operands loaded per slot
constexpr int kSeqBwdOut = 2;       // gradients stored per slot
// Staging buffers of the gradients: a slot's buffer is written again three
// slots later, so a store has two slots' work to finish reading it (with
// two buffers, the plain gradient's warps waited on their stores of two
// slots back: 26% of the sampled stalls on the bf16 throughput workload).
constexpr int kSeqBwdOutBufs = 3;

__host__ __device__ constexpr size_t seq_bwd_warp_bytes(int S, int row_bytes, size_t gap = 0) {
    return (size_t(S) * (kSeqBwdIn * kSeqRows * row_bytes + gap) +
            size_t(kSeqBwdOutBufs) * kSeqBwdOut * kSeqRows * row_bytes + size_t(S) * 8 + 127) / 128 * 128;
}

struct SeqBwdParams {
    BwdParams g;         // operands, gradients, initial state, status word (may be null), decay
    int64_t n_groups;    // channel groups per batch row
    int64_t n_warps;     // B * n_groups
    int slots;           // load ring depth S
};

template <class BOp, typename IO, int WB, bool DT = false>
__global__ void __launch_bounds__(WB * 32)
scan_sequential_backward_kernel(const SeqBwdParams q, const __grid_constant__ CUtensorMap map_in0,
                                const __grid_constant__ CUtensorMap map_in1,
                                const __grid_constant__ CUtensorMap map_gy,
                                const __grid_constant__ CUtensorMap map_fwd,
                                const __grid_constant__ CUtensorMap map_d0,
                                const __grid_constant__ CUtensorMap map_d1,
                                const __grid_constant__ CUtensorMap map_gap) {
    static_assert(!DT || BOp::kDecay, "gaps through the copy engine need a decay operator");
    static_assert(kSeqRows % 2 == 0, "rows are taken in pairs");
    constexpr uint32_t kGap = DT ? kSeqGapBytes : 0;
    using LR = LaneRow<IO>;
    constexpr int CW = 32;
    constexpr int kRowBytes = seq_row_bytes<IO>();
    constexpr uint32_t kOpBytes = kSeqRows * kRowBytes;             // one operand of a slot
    const BwdParams &bp = q.g;
    const ScanParams &p = bp.s;
    extern __shared__ __align__(128) unsigned char smem[];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t gw = int64_t(blockIdx.x) * WB + warp;
    if (gw >= q.n_warps) return;                                     // no block barrier below
    const int S = q.slots;
    const int64_t b = gw / q.n_groups;
    const int64_t grp = gw - b * q.n_groups;
    const int x0 = int(grp) * CW;
    const int64_t d = int64_t(x0) + lane;

    constexpr uint32_t kSlot = kSeqBwdIn * kOpBytes + kGap;         // [in0 | in1 | gy | fwd | gaps]
    const uint32_t base = smem_addr(smem) + uint32_t(warp * seq_bwd_warp_bytes(S, kRowBytes, kGap));
    const uint32_t ring = base;
    const uint32_t outb = base + uint32_t(S) * kSlot;                // 3 x [d in0 | d in1]
    const uint32_t bars = outb + kSeqBwdOutBufs * kSeqBwdOut * kOpBytes;

    const int n_slots = int((p.T + kSeqRows - 1) / kSeqRows);       // T < 2^31 (host check)
    // processing slot i covers time rows [j RB, j RB + RB), j = n_slots - 1 - i
    auto issue = [&](int i, int s) {
        const int y = (n_slots - 1 - i) * kSeqRows;
        const uint32_t dst = ring + uint32_t(s) * kSlot;
        const uint32_t bar = bars + 8u * uint32_t(s);
        mbar_expect_tx(bar, kSeqBwdIn * kOpBytes + (DT ? kSeqRows * 4 : 0));
        tma_load_3d(dst, &map_in0, x0, y, int(b), bar);
        tma_load_3d(dst + kOpBytes, &map_in1, x0, y, int(b), bar);
        tma_load_3d(dst + 2 * kOpBytes, &map_gy, x0, y, int(b), bar);
        tma_load_3d(dst + 3 * kOpBytes, &map_fwd, x0, y - 1, int(b), bar);   // state before each row
        if constexpr (DT) tma_load_2d(dst + kSeqBwdIn * kOpBytes, &map_gap, y, int(b), bar);
    };
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bars + 8u * s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int s = 0; s < S && s < n_slots; ++s) issue(s, s);
    }
    __syncwarp();

    const float h_init =
        (bp.init && d < p.D) ? load_scalar<IO>(static_cast<const IO *>(bp.init) + b * bp.init_bs + d)
                             : BOp::default_state();
    [[maybe_unused]] float lam2 = 0.f, dl = 0.f, gcur = 0.f;
    [[maybe_unused]] float gnext = 0.f;
    if constexpr (BOp::kDecay) {
        lam2 = decay_lam2(p, d);
        if constexpr (!DT) {
            gcur = seq_slot_gap(p, b, int64_t(n_slots - 1) * kSeqRows, lane);
            gnext = seq_slot_gap(p, b, int64_t(n_slots - 2) * kSeqRows, lane);
        }
    }

    float lam = 0.f;           // dL/d (state after the rows still to walk)
    uint32_t wait_limit = kMbarLimit;
    bool bad = false;
    int s = 0;
    uint32_t phase = 0;
    for (int i = 0; i < n_slots; ++i) {
        const int j = n_slots - 1 - i;
        [[maybe_unused]] float gnext2 = 0.f;                        // the gaps two slots below
        if constexpr (BOp::kDecay && !DT) gnext2 = seq_slot_gap(p, b, int64_t(j - 2) * kSeqRows, lane);
        if (!mbar_wait(bars + 8u * uint32_t(s), phase, wait_limit)) {
            wait_limit = 1;
            if (!bad && lane == 0 && p.status) atomicOr(p.status, kTimeoutBit);
            bad = true;
        }
        const uint32_t src = ring + uint32_t(s) * kSlot + uint32_t(lane) * uint32_t(sizeof(IO));
        float xk[kSeqRows], xh[kSeqRows], xg[kSeqRows], xf[kSeqRows];
#pragma unroll
        for (int r = 0; r < kSeqRows; ++r) {
            xk[r] = LR::load(src + r * kRowBytes);
            xh[r] = LR::load(src + kOpBytes + r * kRowBytes);
            xg[r] = LR::load(src + 2 * kOpBytes + r * kRowBytes);
            xf[r] = LR::load(src + 3 * kOpBytes + r * kRowBytes);
        }
        if constexpr (DT) gcur = seq_smem_gap(p, ring + uint32_t(s) * kSlot + kSeqBwdIn * kOpBytes, lane);
        if (lane == 0) bulk_wait_read<kSeqBwdOutBufs - 1>();         // staging buffers of slot i - 3
        __syncwarp();
        if (lane == 0 && !bad && i + S < n_slots) {
            fence_proxy_async();
            issue(i + S, s);
        }
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }
        if (j == 0) xf[0] = h_init;                                  // the state before t = 0
        const uint32_t obuf = outb + uint32_t(i % kSeqBwdOutBufs) * kSeqBwdOut * kOpBytes;
        const uint32_t dst = obuf + uint32_t(lane) * uint32_t(sizeof(IO));
        const int valid = int(p.T - int64_t(j) * kSeqRows);         // rows of the slot inside T (>= 1)
        // rows r and r - 1 as the two halves of packed fp32x2 operations
        // (coefficients, outputs, dL/dlambda terms); the gradient itself
        // runs through them one row at a time
        auto rows = [&](auto fullc) {
            constexpr bool FULL = decltype(fullc)::value;
#pragma unroll
            for (int r = kSeqRows - 1; r >= 1; r -= 2) {
                const float2 k2 = make_float2(xk[r], xk[r - 1]);
                const float2 h2 = make_float2(xh[r], xh[r - 1]);
                const float2 f2 = make_float2(xf[r], xf[r - 1]);
                float2 A, cP, cQ;
                [[maybe_unused]] float2 u2 = make_float2(0.f, 0.f);
                if constexpr (BOp::kDecay) {
                    u2 = make_float2(__shfl_sync(0xffffffffu, gcur, r), __shfl_sync(0xffffffffu, gcur, r - 1));
                    BOp::coeffs_gated2(k2, h2, f2, decay_gamma2(make_float2(lam2, lam2), u2), A, cP, cQ);
                } else {
                    BOp::coeffs2(k2, h2, f2, A, cP, cQ);
                }
                float2 delta, lamn;
                delta.x = xg[r] + lam;
                if (FULL || r < valid) lam = A.x * delta.x;
                lamn.x = lam;
                delta.y = xg[r - 1] + lam;
                if (FULL || r - 1 < valid) lam = A.y * delta.y;
                lamn.y = lam;
                if constexpr (BOp::kDecay) {
                    // dL/dlambda gains delta (1 - z) h_{t-1} dgamma/dlambda
                    //   = delta A h_{t-1} (-u) = (A delta) (-u h_{t-1})
                    float2 e = __fmul2_rn(f2, make_float2(-u2.x, -u2.y));
                    if (!FULL) {
                        if (r >= valid) e.x = 0.f;
                        if (r - 1 >= valid) e.y = 0.f;
                    }
                    const float2 de = __fmul2_rn(lamn, e);
                    dl += de.x + de.y;
                }
                const float2 o0 = __fmul2_rn(delta, cP), o1 = __fmul2_rn(delta, cQ);
                LR::store(dst + r * kRowBytes, o0.x);
                LR::store(dst + (r - 1) * kRowBytes, o0.y);
                LR::store(dst + kOpBytes + r * kRowBytes, o1.x);
                LR::store(dst + kOpBytes + (r - 1) * kRowBytes, o1.y);
            }
        };
        if (__any_sync(0xffffffffu, bad)) {
            // a copy of this or an earlier slot never landed: NaN gradients
            bad = true;
#pragma unroll
            for (int r = 0; r < kSeqRows; ++r) {
                LR::store(dst + r * kRowBytes, __int_as_float(0x7fffffff));
                LR::store(dst + kOpBytes + r * kRowBytes, __int_as_float(0x7fffffff));
            }
        } else if (valid >= kSeqRows) {
            rows(std::true_type{});
        } else {
            rows(std::false_type{});
        }
        fence_proxy_async();                                         // gradients visible to the stores
        __syncwarp();
        if (lane == 0) {
            tma_store_3d(&map_d0, obuf, x0, j * kSeqRows, int(b));
            tma_store_3d(&map_d1, obuf + kOpBytes, x0, j * kSeqRows, int(b));
            bulk_commit();
        }
        if constexpr (BOp::kDecay && !DT) {
            gcur = gnext;
            gnext = gnext2;
        }
    }
    if (bp.dinit && d < p.D) {
        const float y[1] = {bad ? __int_as_float(0x7fffffff) : lam};
        Access<IO, 1>::store(static_cast<IO *>(bp.dinit) + b * bp.dinit_bs + d, y);
    }
    if constexpr (BOp::kDecay) {
        if (bp.dlam && d < p.D) atomicAdd(bp.dlam + d, dl);
    }
    if (lane == 0) bulk_wait_all();
}

}  // namespace sgr
