// projected_scan.cuh -- the minGRU layer's input projection fused with its scan.
//
// The layer (page "Mingru Pytorch": a module applied to a (B, T, d) input)
// computes k and hx from the input by a linear projection and scans them.
// Here one kernel does both for a tile of 64 channels x 256 tokens:
//   k[c, t]  = sum_j W[c, j] x[t, j],   hx[c, t] = sum_j W[D + c, j] x[t, j]
// on the 5th-generation tensor cores (tcgen05.mma, bf16 operands, fp32
// accumulators in tensor memory, operands staged by the tensor memory
// accelerator with 128-byte swizzle), then the activations, the tile's scan
// and the chunk hand-off of the scan engine, and writes h.  k and hx never go
// to HBM.
//
// The product is taken transposed: the MMA's M side is the tile's 64 k rows
// and 64 hx rows of W, interleaved in groups of 16 (W rows k 0-15, hx 0-15,
// k 16-31, hx 16-31, ...), its N side 256 tokens.  Tensor-memory lane = W
// row, column = token, so every thread that reads the accumulator holds one
// channel's values along time -- the order of the recurrence -- and the k and
// hx of a channel sit 16 lanes apart in the same warp, one shuffle from each
// other.  No shared-memory transpose, and one look-back per tile.
//
// Persistent blocks, one per SM (cooperative launch: every look-back waits
// for a block that is resident), each taking tiles blockIdx.x, blockIdx.x +
// gridDim.x, ...  Warp 0 streams W and x tiles by TMA into a 4-stage ring
// (per stage one box of x and one box of W, the latter through a 4-D view of
// W -- (K, row in a 16-row group, k or hx, group) -- that lands the tile's
// rows in the interleaved order above; issuing the W rows as eight 16-row
// boxes instead measured 11% slower)
// (continuing across tiles); one thread of warp 1 issues the MMAs of tile i
// into one of two accumulators (512 tensor-memory columns in all) while warps
// 4-19 run the epilogue of tile i-1 from the other.  Epilogue warp (q, g)
// reads lane quarter q (channels 16q .. 16q+15, k and hx) and columns 64g ..
// 64g+63; after the exchange each thread owns one channel and 32 consecutive
// tokens: it computes their (a, b) pairs into registers and folds them; warp
// 2 combines the eight folds of each channel, publishes the chunk summary,
// looks back and publishes the state; each thread then replays its tokens
// from the state before them and stores h.  The carry is warp 2's, so that the
// look-back's registers do not add to the epilogue threads' (which hold their
// 32 pairs across it).
#pragma once

#include "scan_engine.cuh"

namespace sgr {

struct ProjParams {
    ScanParams s;        // B, T, D, chunk/chain counts, hand-off words, status; out = h (fp32),
                         // init = h0 (fp32 rows) or null
    int64_t d_in;        // projection input width (multiple of 64)
};

namespace proj {

constexpr int kTR = 256;            // tokens per tile (MMA N)
constexpr int kTC = 64;             // channels per tile
constexpr int kM = 2 * kTC;         // MMA M: k and hx rows of W
constexpr int kGrp = 16;            // W rows per interleave group
constexpr int kKB = 64;             // K per stage: one 128-byte swizzle row of bf16
constexpr int kStages = 4;
constexpr uint32_t kGrpBytes = kGrp * kKB * 2;  // 2 KB: one group of W rows
constexpr uint32_t kABytes = kM * kKB * 2;      // 16 KB (W)
constexpr uint32_t kBBytes = kTR * kKB * 2;     // 32 KB (x)
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kRingBytes = kStages * kStageBytes;            // 192 KB
constexpr uint32_t kBarOffset = kRingBytes;
constexpr int kEpiWarps = 16;                   // warps 4 .. 19
constexpr int kThreads = (4 + kEpiWarps) * 32;
constexpr int kSegs = kEpiWarps / 4 * 2;        // 32-token segments of a tile: 8
// + align slack; barriers; per tile parity: the segments' folds and the
// channels' incoming states
constexpr uint32_t kSmemBytes = 1024 + kBarOffset + 256 + 2 * kSegs * kTC * 8 + 2 * kTC * 4;
static_assert(kSmemBytes <= 227 * 1024, "one block per SM");
static_assert(kSegs * 32 == kTR && kEpiWarps % 4 == 0, "epilogue covers the tile");
constexpr uint32_t kAccCols = kTR;              // fp32 accumulator columns per tile
constexpr uint32_t kTmemCols = 2 * kAccCols;    // two accumulators
constexpr uint32_t kWaitLimit = 1u << 20;

// K-major operand with 128-byte swizzle: rows of 128 bytes, 8-row groups
// 1024 bytes apart (tcgen05 shared-memory matrix descriptor, version 1)
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
    uint64_t d = uint64_t((addr >> 4) & 0x3FFF);
    d |= uint64_t(1) << 16;            // leading byte offset (unused with this swizzle)
    d |= uint64_t(1024 >> 4) << 32;    // stride byte offset
    d |= uint64_t(1) << 46;            // descriptor version
    d |= uint64_t(2) << 61;            // 128-byte swizzle
    return d;
}

// kind::f16 instruction descriptor: bf16 x bf16 -> fp32, both K-major, M x N
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kTR >> 3) << 17) |
                            (uint32_t(kM >> 4) << 24);

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int x, int y, int z, int w,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar) : "memory");
}

// bounded wait; false if the phase did not complete
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// 32 consecutive accumulator columns of this thread's lane (lane quarter of
// the warp); completes with tmem_wait
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

}  // namespace proj

__global__ void __launch_bounds__(proj::kThreads, 1) mingru_projected_scan_kernel(
    const ProjParams pp, const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w) {
    using namespace proj;
    using Op = MinGRUOp;
    constexpr int CV = kTC / 32;            // channels per carry lane
    const ScanParams &p = pp.s;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                            ~uintptr_t(1023));
    // full[S], empty[S], acc_full[2], acc_empty[2]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOffset);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kStages + 4);
    float2 *s_part = reinterpret_cast<float2 *>(smem + kBarOffset + 256);              // [2][kSegs][kTC]
    float *s_hin = reinterpret_cast<float *>(smem + kBarOffset + 256 + 2 * kSegs * kTC * 8);  // [2][kTC]
    const uint32_t ring = smem_addr(smem);
    auto full = [&](int s) { return smem_addr(&bars[s]); };
    auto empty = [&](int s) { return smem_addr(&bars[kStages + s]); };
    auto acc_full = [&](int a) { return smem_addr(&bars[2 * kStages + a]); };
    auto acc_empty = [&](int a) { return smem_addr(&bars[2 * kStages + 2 + a]); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t G = gridDim.x;
    const int64_t first = blockIdx.x;
    const int n_local = int((p.n_tiles - first + G - 1) / G);
    const int n_kb = int(pp.d_in / kKB);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 * kStages + 2; ++i) mbar_init(smem_addr(&bars[i]), 1);
        // each epilogue warp hands the accumulator back once it has read its part
        for (int i = 2 * kStages + 2; i < 2 * kStages + 4; ++i) mbar_init(smem_addr(&bars[i]), kEpiWarps);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(tmem_slot)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // producer: for each tile, the W rows of channels [dt kTC, +kTC) in
            // interleaved groups (group gi of kind k, k = 0 for k rows, 1 for
            // hx rows, goes to A row (2 gi + k) kGrp) and x rows [c kTR, +kTR)
            // of batch row b; K in steps of kKB
            bool ok = true;
            int64_t g = 0;                               // K steps issued so far
            for (int n = 0; n < n_local && ok; ++n) {
                const TileCoord tc = tile_coord(p, uint32_t(first + int64_t(n) * G));
                const int w_row = int(int64_t(tc.dt) * kTC);
                for (int kb = 0; kb < n_kb; ++kb, ++g) {
                    const int s = int(g % kStages);
                    if (g >= kStages && !wait(empty(s), uint32_t((g / kStages - 1) & 1), kWaitLimit)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = ring + uint32_t(s) * kStageBytes;
                    mbar_expect_tx(full(s), kStageBytes);
                    // W viewed as (K, row in group, k/hx, group): one box of
                    // (kKB, kGrp, 2, kTC / kGrp) lands in the interleaved order
                    tma_load_4d(a_dst, &map_w, kb * kKB, 0, 0, w_row / kGrp, full(s));
                    tma_load_3d(a_dst + kABytes, &map_x, kb * kKB, int(tc.c) * kTR, int(tc.b), full(s));
                }
            }
            if (!ok) atomicOr(p.status, kTimeoutBit);
            // a block never leaves with copies in flight: wait (bounded) for the
            // last stages issued, which the MMA thread also waits for
            for (int64_t k = g > kStages ? g - kStages : 0; k < g; ++k)
                wait(full(int(k % kStages)), uint32_t((k / kStages) & 1), kWaitLimit);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // MMA issuer: tile n into accumulator n & 1 once the epilogue has read it
            bool ok = true;
            int64_t g = 0;
            for (int n = 0; n < n_local && ok; ++n) {
                const int a = n & 1;
                if (n >= 2 && !wait(acc_empty(a), uint32_t((n / 2 - 1) & 1), kWaitLimit)) {
                    ok = false;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;");
                const uint32_t acc = tmem + uint32_t(a) * kAccCols;
                for (int kb = 0; kb < n_kb; ++kb, ++g) {
                    const int s = int(g % kStages);
                    if (!wait(full(s), uint32_t((g / kStages) & 1), kWaitLimit)) {
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;");
                    const uint32_t a_addr = ring + uint32_t(s) * kStageBytes;
                    const uint64_t da = sw128_desc(a_addr), db = sw128_desc(a_addr + kABytes);
#pragma unroll
                    for (int kk = 0; kk < kKB / 16; ++kk) {
                        const uint32_t accumulate = (kb > 0 || kk > 0) ? 1u : 0u;
                        asm volatile(
                            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                            ::"r"(acc), "l"(da + uint64_t(kk * 2)), "l"(db + uint64_t(kk * 2)), "r"(kIdesc),
                              "r"(accumulate));
                    }
                    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                                 ::"r"(empty(s)) : "memory");
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                             ::"r"(acc_full(a)) : "memory");
            }
            if (!ok) atomicOr(p.status, kTimeoutBit);
        }
        __syncwarp();
    } else if (warp == 2) {
        // the carry warp: for each tile, the chunk hand-off of the scan engine
        // (publish the summary, look back, publish the state) for the tile's
        // channels, CV per lane, from the epilogue's segment folds
        constexpr uint32_t NE = kEpiWarps * 32;
        const int cl = lane * CV;
        for (int n = 0; n < n_local; ++n) {
            const int64_t tile = first + int64_t(n) * G;
            const TileCoord tc = tile_coord(p, uint32_t(tile));
            const int64_t c = tc.c, b = tc.b, dt = tc.dt, chain = tc.chain;
            const float2 *part = s_part + (n & 1) * kSegs * kTC;
            float *hin_s = s_hin + (n & 1) * kTC;
            named_barrier_sync(1, NE + 32);
            float2 total[CV];
#pragma unroll
            for (int v = 0; v < CV; ++v) {
                total[v] = part[cl + v];
#pragma unroll
                for (int sg = 1; sg < kSegs; ++sg) total[v] = Op::combine(total[v], part[sg * kTC + cl + v]);
            }
            const bool publish = (p.n_chunks > 1) && (int64_t(c) < p.n_chunks - 1) && (tile != p.drop_tile);
            const int64_t dl = dt * kTC + cl;
            float hin[CV];
            if (c == 0) {
#pragma unroll
                for (int v = 0; v < CV; ++v) hin[v] = load_init<float>(p, b, dl + v, Op::default_init());
            } else {
                if (publish) publish_summary<CV, kTC>(p, tile, cl, total);
                look_back<Op, float, CV, kTC>(p, c, chain, b, dl, cl, hin);
            }
#pragma unroll
            for (int v = 0; v < CV; ++v) hin_s[cl + v] = hin[v];
            __syncwarp();
            named_barrier_arrive(2, NE + 32);
            if (publish) {
                float fin[CV];
#pragma unroll
                for (int v = 0; v < CV; ++v) fin[v] = Op::apply(total[v], hin[v]);
                publish_state<CV, kTC>(p, tile, cl, fin);
            }
        }
    } else if (warp >= 4) {
        // epilogue
        constexpr uint32_t NE = kEpiWarps * 32;
        const int q = warp & 3;                      // lane quarter: channels 16q .. 16q+15
        const int cg = (warp - 4) >> 2;              // column group: tokens 64 cg .. 64 cg + 63
        const bool hx_lane = lane >= 16;             // this lane reads hx (else k)
        const int ch = q * kGrp + (lane & 15);       // channel within the tile
        const int seg = 2 * cg + (hx_lane ? 1 : 0);  // 32-token segment this thread scans
        const int tok0 = seg * 32;
        for (int n = 0; n < n_local; ++n) {
            const int64_t tile = first + int64_t(n) * G;
            const TileCoord tc = tile_coord(p, uint32_t(tile));
            const int64_t c = tc.c, b = tc.b, dt = tc.dt;
            const int a = n & 1;
            float2 *part = s_part + a * kSegs * kTC;
            float *hin_s = s_hin + a * kTC;
            if (!wait(acc_full(a), uint32_t((n / 2) & 1), kWaitLimit)) atomicOr(p.status, kTimeoutBit);
            __syncwarp();                            // tensor-memory loads are warp-collective
            asm volatile("tcgen05.fence::after_thread_sync;");
            uint32_t r0[32], r1[32];
            const uint32_t taddr = tmem + (uint32_t(q * 32) << 16) + uint32_t(a) * kAccCols + uint32_t(cg * 64);
            tmem_ld32(taddr, r0);
            tmem_ld32(taddr + 32, r1);
            tmem_wait();
            asm volatile("tcgen05.fence::before_thread_sync;");
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acc_empty(a)) : "memory");

            // k lanes keep columns 0-31 of the group and take hx of them from the
            // partner lane; hx lanes keep columns 32-63 and take k of them
            const int rows = int(p.T - c * kTR < kTR ? p.T - c * kTR : kTR);
            float av[32], bv[32];
            float2 fold = Op::identity();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float sent = __uint_as_float(hx_lane ? r0[i] : r1[i]);
                const float got = __shfl_xor_sync(0xffffffffu, sent, 16);
                const float kv = hx_lane ? got : __uint_as_float(r0[i]);
                const float hv = hx_lane ? __uint_as_float(r1[i]) : got;
                float x = 1.f, y = 0.f;              // tokens past T: the identity pair
                if (tok0 + i < rows) Op::element(kv, hv, x, y);
                av[i] = x;
                bv[i] = y;
                fold = Op::combine(fold, make_float2(x, y));
            }
            part[seg * kTC + ch] = fold;
            named_barrier_arrive(1, NE + 32);        // the folds are in shared memory
            named_barrier_sync(2, NE + 32);          // the carry warp has written the states
            // replay this thread's tokens from the state before them and store h
            float st = hin_s[ch];
            for (int sg = 0; sg < seg; ++sg) st = Op::apply(part[sg * kTC + ch], st);
            float *out = static_cast<float *>(p.out) + (b * p.T + c * kTR + tok0) * p.D + dt * kTC + ch;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                st = Op::step(av[i], bv[i], st);
                if (tok0 + i < rows) __stcs(out + int64_t(i) * p.D, st);
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

}  // namespace sgr
