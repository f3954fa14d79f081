// projected_scan.cuh -- the minGRU layer's input projection fused with its scan.
//
// The layer (page "Mingru Pytorch": a module applied to a (B, T, d) input)
// computes k and hx from the input by a linear projection and scans them.
// Here one kernel does both for a tile of 128 tokens x 128 channels:
//   k[t, c]  = sum_j x[t, j] W[c, j],   hx[t, c] = sum_j x[t, j] W[D + c, j]
// on the 5th-generation tensor cores (tcgen05.mma, bf16 operands, fp32
// accumulators in tensor memory, operands staged by the tensor memory
// accelerator with 128-byte swizzle), then the activations, the tile's scan
// and the chunk hand-off of the scan engine, and writes h.  k and hx never go
// to HBM.
//
// Warp roles (8 warps): warp 0 loads x and W tiles into a 2-stage ring; warp
// 1 allocates tensor memory and issues the MMAs (one thread); then all 8
// warps run the epilogue, for each half of the tile's channels in turn: each
// thread reads 32 accumulator columns of one token row and writes the (a, b)
// pairs to shared memory (the ring, idle by then), then owns one channel and
// a quarter of the rows: folds them, gets the tile's incoming state (warp 0
// publishes the chunk summary and looks back), replays and stores.  About 99 KB of
// shared memory and 256 of the 512 tensor-memory columns per block, so two
// blocks share an SM and one's epilogue runs beside the other's MMAs.
#pragma once

#include "scan_engine.cuh"

namespace sgr {

struct ProjParams {
    ScanParams s;        // B, T, D, chunk/chain counts, hand-off words, status; out = h (fp32),
                         // init = h0 (fp32 rows) or null
    int64_t d_in;        // projection input width (multiple of 64)
};

namespace proj {

constexpr int kTR = 128;            // tokens per tile (MMA M)
constexpr int kTC = 128;            // channels per tile: N = 2 kTC (k and hx)
constexpr int kN = 2 * kTC;
constexpr int kKB = 64;             // K per stage: one 128-byte swizzle row of bf16
constexpr int kStages = 2;          // two blocks per SM: one's epilogue overlaps the other's MMAs
constexpr int kHalf = kTC / 2;      // the epilogue handles the channels in two halves
constexpr uint32_t kABytes = kTR * kKB * 2;     // 16 KB
constexpr uint32_t kBBytes = kN * kKB * 2;      // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kRingBytes = kStages * kStageBytes;            // 96 KB
constexpr uint32_t kPairBytes = kTR * kHalf * 8;                  // 64 KB, aliases the ring
static_assert(kPairBytes <= kRingBytes, "pairs fit in the idle ring");
constexpr uint32_t kBarOffset = kRingBytes;
// + align slack; barriers; four row-quarter fold results and the incoming states
constexpr uint32_t kSmemBytes = 1024 + kRingBytes + 256 + 4 * kHalf * 8 + kHalf * 4;
constexpr uint32_t kTmemCols = 256;
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
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kN >> 3) << 17) |
                            (uint32_t(kTR >> 4) << 24);

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}

// bounded wait; false if the phase did not complete
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// 32 consecutive accumulator columns of this thread's row (lane quarter of
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

// the pair of (row r, channel c of the half) in the epilogue buffer: rows of
// kHalf pairs, channel index xor-ed with the row's low bits so that a warp
// writing one channel of 32 rows, and a warp reading 32 channels of one row,
// both touch every bank evenly
__device__ __forceinline__ uint32_t pair_slot(int r, int c) { return uint32_t(r * kHalf + (c ^ (r & 15))); }

}  // namespace proj

__global__ void __launch_bounds__(256, 2) mingru_projected_scan_kernel(const ProjParams pp,
                                                                      const __grid_constant__ CUtensorMap map_x,
                                                                      const __grid_constant__ CUtensorMap map_w) {
    using namespace proj;
    using Op = MinGRUOp;
    constexpr int CV = kHalf / 32;          // channels per carry lane within a half
    const ScanParams &p = pp.s;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                            ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOffset);   // full[S], empty[S], done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kStages + 1);
    float2 *s_part = reinterpret_cast<float2 *>(smem + kBarOffset + 256);          // [4][kHalf]
    float *s_hin = reinterpret_cast<float *>(smem + kBarOffset + 256 + 4 * kHalf * 8);
    float2 *pairs = reinterpret_cast<float2 *>(smem);                   // after the MMAs: the ring's space
    const uint32_t ring = smem_addr(smem);
    auto full = [&](int s) { return smem_addr(&bars[s]); };
    auto empty = [&](int s) { return smem_addr(&bars[kStages + s]); };
    const uint32_t done = smem_addr(&bars[2 * kStages]);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tile = blockIdx.x;
    const TileCoord tc = tile_coord(p, uint32_t(tile));
    const int64_t c = tc.c, b = tc.b, ct = tc.dt, chain = tc.chain;
    const int n_kb = int(pp.d_in / kKB);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 * kStages + 1; ++i) mbar_init(smem_addr(&bars[i]), 1);
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

    if (warp == 0 && lane == 0) {
        // producer: x rows [c kTR, c kTR + kTR) of batch row b; W rows
        // [ct kTC, +kTC) (k) and [D + ct kTC, +kTC) (hx); K in steps of kKB
        bool ok = true;
        for (int kb = 0; kb < n_kb && ok; ++kb) {
            const int s = kb % kStages;
            if (kb >= kStages && !wait(empty(s), uint32_t((kb / kStages - 1) & 1), kWaitLimit)) {
                ok = false;
                break;
            }
            const uint32_t a_dst = ring + uint32_t(s) * kStageBytes;
            const uint32_t b_dst = a_dst + kABytes;
            mbar_expect_tx(full(s), kStageBytes);
            tma_load_3d(a_dst, &map_x, kb * kKB, int(c) * kTR, int(b), full(s));
            tma_load_2d(b_dst, &map_w, kb * kKB, int(ct) * kTC, full(s));
            tma_load_2d(b_dst + kBBytes / 2, &map_w, kb * kKB, int(p.D + ct * kTC), full(s));
        }
        if (!ok) atomicOr(p.status, kTimeoutBit);
    } else if (warp == 1 && lane == 0) {
        // MMA issuer
        bool ok = true;
        for (int kb = 0; kb < n_kb; ++kb) {
            const int s = kb % kStages;
            if (!wait(full(s), uint32_t((kb / kStages) & 1), kWaitLimit)) {
                ok = false;
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;");
            const uint32_t a_addr = ring + uint32_t(s) * kStageBytes;
            const uint64_t da = sw128_desc(a_addr), db = sw128_desc(a_addr + kABytes);
#pragma unroll
            for (int kk = 0; kk < kKB / 16; ++kk) {
                const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
                asm volatile(
                    "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                    ::"r"(tmem), "l"(da + uint64_t(kk * 2)), "l"(db + uint64_t(kk * 2)), "r"(kIdesc), "r"(acc));
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         ::"r"(empty(s)) : "memory");
        }
        if (!ok) atomicOr(p.status, kTimeoutBit);
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                     ::"r"(done) : "memory");
    }
    __syncwarp();        // lanes 1-31 of warps 0 and 1 wait here for their lane 0's role
    {
        // epilogue, all 8 warps (the producer and MMA threads have issued
        // everything by now).  Warp w reads tensor-memory lane quarter w % 4
        // (token rows 32 (w % 4) ..) and, of each half of the channels, the
        // 32 columns w / 4.
        constexpr uint32_t NE = 256;
        const int q = warp & 3;
        const int cs = warp >> 2;
        const int r = q * 32 + lane;                 // this thread's token row
        const int64_t t = c * kTR + r;
        if (!wait(done, 0, kWaitLimit)) atomicOr(p.status, kTimeoutBit);
        __syncwarp();    // tensor-memory loads are warp-collective
        asm volatile("tcgen05.fence::after_thread_sync;");
        // every TMA load has landed and every MMA has read its operands: the
        // ring's space now holds the pairs, one half of the channels at a time
        const bool valid = t < p.T;
        const int ch = threadIdx.x & (kHalf - 1);    // fold and replay: channel of the half ...
        const int rq = threadIdx.x / kHalf;          // ... and quarter of the rows
        const int rows = int(p.T - c * kTR < kTR ? p.T - c * kTR : kTR);
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
            {
                // k and hx of 32 channels of this row: both loads in flight, one wait
                uint32_t kv[32], hv[32];
                tmem_ld32(tmem + (uint32_t(q * 32) << 16) + uint32_t(hf * kHalf + cs * 32), kv);
                tmem_ld32(tmem + (uint32_t(q * 32) << 16) + uint32_t(kTC + hf * kHalf + cs * 32), hv);
                tmem_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float a = 1.f, bb = 0.f;         // rows past T: the identity pair
                    if (valid) Op::element(__uint_as_float(kv[i]), __uint_as_float(hv[i]), a, bb);
                    pairs[pair_slot(r, cs * 32 + i)] = make_float2(a, bb);
                }
            }
            named_barrier_sync(1, NE);
            // fold this thread's 32 rows of its channel
            float2 part = Op::identity();
#pragma unroll 8
            for (int rr = rq * 32; rr < rq * 32 + 32; ++rr) part = Op::combine(part, pairs[pair_slot(rr, ch)]);
            s_part[rq * kHalf + ch] = part;
            named_barrier_sync(2, NE);
            if (warp == 0) {
                // the chunk hand-off (scan engine): publish the summary, look back, publish the state
                const int cl = lane * CV;                 // channel within the half
                const int ct_ch = hf * kHalf + cl;        // channel within the tile
                float2 total[CV];
#pragma unroll
                for (int v = 0; v < CV; ++v) {
                    total[v] = s_part[cl + v];
#pragma unroll
                    for (int qq = 1; qq < 4; ++qq) total[v] = Op::combine(total[v], s_part[qq * kHalf + cl + v]);
                }
                const bool publish = (p.n_chunks > 1) && (c < p.n_chunks - 1) && (tile != p.drop_tile);
                const int64_t dl = ct * kTC + ct_ch;
                float hin[CV];
                if (c == 0) {
#pragma unroll
                    for (int v = 0; v < CV; ++v) hin[v] = load_init<float>(p, b, dl + v, Op::default_init());
                } else {
                    if (publish) publish_summary<CV, kTC>(p, tile, ct_ch, total);
                    look_back<Op, float, CV, kTC>(p, c, chain, b, dl, ct_ch, hin);
                }
#pragma unroll
                for (int v = 0; v < CV; ++v) s_hin[cl + v] = hin[v];
                if (publish) {
                    float fin[CV];
#pragma unroll
                    for (int v = 0; v < CV; ++v) fin[v] = Op::apply(total[v], hin[v]);
                    publish_state<CV, kTC>(p, tile, ct_ch, fin);
                }
            }
            named_barrier_sync(3, NE);
            // replay the channel's rows from their incoming state and store h
            float st = s_hin[ch];
            for (int qq = 0; qq < rq; ++qq) st = Op::apply(s_part[qq * kHalf + ch], st);
            float *out = static_cast<float *>(p.out) + (b * p.T + c * kTR) * p.D + ct * kTC + hf * kHalf + ch;
            const int r1 = rq * 32 + 32 < rows ? rq * 32 + 32 : rows;
#pragma unroll 4
            for (int rr = rq * 32; rr < r1; ++rr) {
                const float2 pr = pairs[pair_slot(rr, ch)];
                st = Op::step(pr.x, pr.y, st);
                __stcs(out + int64_t(rr) * p.D, st);
            }
            named_barrier_sync(1, NE);                   // the buffer is free for the next half
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
