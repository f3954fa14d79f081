// scan_pipelined_backward.cuh -- the gradients of both scans on persistent,
// copy-engine-fed blocks, for aligned rows of narrow batches (where the
// channel groups alone do not fill the GPU and the time axis is cut into
// chunks).
//
// The gradient is the reverse-time affine recurrence of scan_backward.cuh:
// with lam the gradient reaching out_t from the steps after t,
//   delta_t = gy_t + lam,  d in0_t = delta_t cP_t,  d in1_t = delta_t cQ_t,
//   lam <- A_t delta_t = A_t lam + A_t gy_t,
// the pair (A_t, A_t gy_t) composed in reverse time.  Chunks are numbered in
// processing order (processing chunk c covers time chunk n_chunks - 1 - c),
// so the scan engine's chunk hand-off and look-back carry lam unchanged.
//
// Layout, as the forward pipelined kernel's: persistent co-resident blocks
// (cooperative launch) of W data warps + 1 carry warp, each owning tiles
// blockIdx.x, blockIdx.x + gridDim.x, ... in order; a tile is TR x TC with
// TC = CG V channels and TR = W J R rows.  Per tile the copy engine brings
// four boxes into a ring slot -- k (or r), hx (or s), dL/dh and the forward
// output starting one row earlier (the state before each row; the row before
// t = 0 reads as zero fill and is replaced by the initial state) -- and, for
// time decay, the tile's rates and gaps.  No multicast.
//
// Data warps: lane (g, j) of warp w owns channels [g V, g V + V) of the
// processing rows [(w J + j) R, (w J + j) R + R); processing row rho of the
// tile is time row ct TR + TR - 1 - rho, which the slot holds at row
// TR - 1 - rho.  Phase A: the local partials (A, cP, cQ) of every element and
// the pair (A, A gy), the fold of the thread's R rows, the scan across the
// warp's J row groups and the warp summary, as in the forward kernel; the
// arithmetic runs on pairs of neighbouring channels (packed fp32x2).  The
// four values per element (A, gy, cP, cQ; with decay also the dL/dlambda
// factor -u h_{t-1}) stay in registers, so phase B of a tile follows its own
// phase A (no one-tile lag): replay lam from the thread's incoming gradient,
// write both input gradients with streaming stores, the initial state's
// gradient from the thread that ends at time row 0, and the dL/dlambda
// terms, summed over the tile in shared memory and added with one atomic
// per channel and tile.  Carry warp: the forward kernel's, with the affine
// operator.
#pragma once

#include "scan_backward.cuh"
#include "scan_engine.cuh"

namespace sgr {

constexpr int kBwdOperands = 4;

template <typename IO, int V, int CG, int R, int S, int W, bool DEC = false>
struct PipeBwdShape {
    static constexpr int J = 32 / CG;
    static constexpr int TC = CG * V;
    static constexpr int TR = W * J * R;
    static constexpr size_t op_bytes = size_t(TR) * TC * sizeof(IO);     // one operand of a tile
    // decay through the copy engine: the tile's TC rates, then its TR gaps
    static constexpr bool dec_boxable = TR % 4 == 0 && TR <= 256 && TC <= 256 && (TC * 4) % 128 == 0;
    static_assert(op_bytes % 128 == 0, "operand copies land on 128-byte boundaries");
    static constexpr size_t dec_bytes = DEC ? size_t(TR + TC) * sizeof(float) : 0;
    static constexpr size_t tx_bytes = kBwdOperands * op_bytes + dec_bytes;
    static constexpr size_t slot_bytes = (tx_bytes + 127) / 128 * 128;
    static constexpr size_t bar_offset = S * slot_bytes;
    static constexpr size_t cnt_offset = bar_offset + S * 8;          // per-slot reader counts
    static constexpr size_t tot_offset = (cnt_offset + S * 4 + 15) / 16 * 16;        // [2][W][TC] float2
    static constexpr size_t total_offset = tot_offset + size_t(2) * W * TC * sizeof(float2);  // [2][TC] float2
    static constexpr size_t hin_offset = total_offset + size_t(2) * TC * sizeof(float2);     // [2][TC] float
    // time decay (with or without its operands through the copy engine): the
    // tile's dL/dlambda sums and their warp count; reserved in every layout
    static constexpr size_t dl_offset = hin_offset + size_t(2) * TC * sizeof(float);        // [2][TC] float
    static constexpr size_t dcnt_offset = dl_offset + size_t(2) * TC * sizeof(float);      // [2] uint
    static constexpr size_t smem_bytes = dcnt_offset + 16;
};

// DT (time decay only): the tile's rates and gaps come with the tile through
// the copy engine (map_lam: the (D,) rates, map_gap: the (B, T) gaps);
// otherwise they are plain loads and the two maps are unused.
template <class BOp, typename IO, int V, int CG, int R, int S, int W, int MINB, bool DT = false>
__global__ void __launch_bounds__((W + 1) * 32, MINB)
scan_pipelined_backward_kernel(const BwdParams bp, const __grid_constant__ CUtensorMap map_in0,
                               const __grid_constant__ CUtensorMap map_in1,
                               const __grid_constant__ CUtensorMap map_gy,
                               const __grid_constant__ CUtensorMap map_fwd,
                               const __grid_constant__ CUtensorMap map_gap,
                               const __grid_constant__ CUtensorMap map_lam) {
    static_assert(!DT || BOp::kDecay, "decay operands through the copy engine need a decay operator");
    using Shape = PipeBwdShape<IO, V, CG, R, S, W, DT>;
    static_assert(!DT || Shape::dec_boxable, "decay operands fit copy boxes");
    static_assert(!DT || (V == 4 && R % 2 == 0), "vector reads of the rates and gaps");
    using Op = MinGRUOp;                 // affine pairs carry the gradient
    using Vec = typename VecOf<IO, V>::type;
    constexpr int J = Shape::J;
    constexpr int TC = Shape::TC;
    constexpr int TR = Shape::TR;
    constexpr int CV = TC / 32;
    constexpr int V2 = V / 2;                 // channel pairs of a thread (packed fp32x2 work)
    constexpr uint32_t NT = (W + 1) * 32;
    constexpr bool kDec = BOp::kDecay;
    // as in the forward kernel: fp32 I/O folds the warp summaries in the last
    // data warp, bf16 I/O in the carry warp
    constexpr bool kFoldInData = sizeof(IO) == 4;
    static_assert(sizeof(Vec) == V * sizeof(IO), "vector type matches the vector width");
    static_assert(CG * J == 32 && TC % 32 == 0, "lane layout");
    static_assert(TC * sizeof(IO) % 16 == 0 && TC <= 256 && TR <= 256, "TMA box");

    const ScanParams &p = bp.s;
    extern __shared__ __align__(128) unsigned char smem[];
    float2 (*s_tot)[W][TC] = reinterpret_cast<float2 (*)[W][TC]>(smem + Shape::tot_offset);
    float2 (*s_total)[TC] = reinterpret_cast<float2 (*)[TC]>(smem + Shape::total_offset);
    float (*s_hin)[TC] = reinterpret_cast<float (*)[TC]>(smem + Shape::hin_offset);
    unsigned int *s_cnt = reinterpret_cast<unsigned int *>(smem + Shape::cnt_offset);
    // time decay: the tile's dL/dlambda, summed over the warps in shared memory
    // and added to the global sums by the last warp to finish the tile
    [[maybe_unused]] float (*s_dl)[TC] = reinterpret_cast<float (*)[TC]>(smem + Shape::dl_offset);
    [[maybe_unused]] unsigned int *s_dcnt = reinterpret_cast<unsigned int *>(smem + Shape::dcnt_offset);
    const uint32_t ring = smem_addr(smem);
    const uint32_t bars = ring + uint32_t(Shape::bar_offset);

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t G = gridDim.x;
    const int64_t first = blockIdx.x;
    const int n_local = int((p.n_tiles - first + G - 1) / G);

    // TMA copies of tile n into ring slot n % S (one thread): the four
    // operands of time chunk ct, the forward output one row earlier
    auto issue_tile = [&](int n) {
        const TileCoord tc = tile_coord(p, uint32_t(first + int64_t(n) * G));
        const int ct = int(p.n_chunks - 1 - int64_t(tc.c));
        const uint32_t slot = ring + uint32_t((n % S) * Shape::slot_bytes);
        const uint32_t bar = bars + 8u * uint32_t(n % S);
        const uint32_t ob = uint32_t(Shape::op_bytes);
        const int x = int(tc.dt) * TC, y = ct * TR, z = int(tc.b);
        mbar_expect_tx(bar, uint32_t(Shape::tx_bytes));
        tma_load_3d(slot, &map_in0, x, y, z, bar);
        tma_load_3d(slot + ob, &map_in1, x, y, z, bar);
        tma_load_3d(slot + 2 * ob, &map_gy, x, y, z, bar);
        tma_load_3d(slot + 3 * ob, &map_fwd, x, y - 1, z, bar);          // the state before each row
        if constexpr (DT) {
            tma_load_1d(slot + 4 * ob, &map_lam, x, bar);
            tma_load_2d(slot + 4 * ob + uint32_t(TC) * 4u, &map_gap, y, z, bar);
        }
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(bars + 8u * s, 1);
            s_cnt[s] = 0;
        }
        if constexpr (BOp::kDecay) {
            for (int i = 0; i < 2 * TC; ++i) (&s_dl[0][0])[i] = 0.f;
            s_dcnt[0] = s_dcnt[1] = 0;
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (warp == W && lane == 0) {
        for (int s = 0; s < S && s < n_local; ++s) issue_tile(s);
    }

    if (warp < W) {
        // ============================================== data warps
        const int g = lane % CG;
        const int j = lane / CG;
        const int rho0 = (warp * J + j) * R;                         // first processing row of the thread
        IO *out0 = static_cast<IO *>(p.out);
        IO *out1 = static_cast<IO *>(bp.out1);
        uint32_t wait_limit = kMbarLimit;
        for (int n = 0; n < n_local; ++n) {
            const int BUF = n & 1;
            const int64_t tile = first + int64_t(n) * G;
            const TileCoord tc = tile_coord(p, uint32_t(tile));
            const int64_t ct = p.n_chunks - 1 - int64_t(tc.c);
            const int64_t d0 = int64_t(tc.dt) * TC + g * V;
            const bool dvalid = d0 < p.D;
            const int64_t top = ct * TR + TR - 1 - rho0;             // time row of r = 0 (>= 0)
            const int64_t base = (int64_t(tc.b) * p.T) * p.D + d0;
            // plain loads issued before the wait: the initial state where the
            // thread ends at time row 0; without the copy engine, the decay
            // rates and gaps
            float h0v[V];
#pragma unroll
            for (int v = 0; v < V; ++v) h0v[v] = BOp::default_state();
            if (bp.init && dvalid && top < R) {
#pragma unroll
                for (int v = 0; v < V; ++v)
                    h0v[v] = load_scalar<IO>(static_cast<const IO *>(bp.init) + int64_t(tc.b) * bp.init_bs + d0 + v);
            }
            [[maybe_unused]] float lam2[V], ur[R];
            if constexpr (kDec && !DT) {
#pragma unroll
                for (int v = 0; v < V; ++v) lam2[v] = decay_lam2(p, d0 + v);
#pragma unroll
                for (int r = 0; r < R; ++r) ur[r] = top - r < p.T ? decay_u(p, tc.b, top - r) : 0.f;
            }
            if (!mbar_wait(bars + 8u * uint32_t(n % S), uint32_t((n / S) & 1), wait_limit)) {
                wait_limit = 1;
                if (lane == 0 && p.status) atomicOr(p.status, kTimeoutBit);
            }
            // the thread's rows in the slot, processing row rho at slot row TR - 1 - rho
            const unsigned char *slot = smem + (n % S) * Shape::slot_bytes;
            const IO *t0 = reinterpret_cast<const IO *>(slot) + (TR - 1 - rho0) * TC + g * V;
            const IO *t1 = t0 + TR * TC;
            const IO *tg = t0 + 2 * TR * TC;
            const IO *tf = t0 + 3 * TR * TC;
            [[maybe_unused]] const float *s_lam = reinterpret_cast<const float *>(slot + 4 * Shape::op_bytes);
            [[maybe_unused]] const float *s_gap = s_lam + TC;
            if constexpr (DT) {
                // the thread's V rates in one shared load, its R gaps (slot rows
                // TR - R - rho0 .. TR - 1 - rho0, R | TR) in R / 2 or one
                const float4 lv = *reinterpret_cast<const float4 *>(s_lam + g * V);
                lam2[0] = lv.x * kNegLog2e;
                lam2[1] = lv.y * kNegLog2e;
                lam2[2] = lv.z * kNegLog2e;
                lam2[3] = lv.w * kNegLog2e;
                const float *gp = s_gap + (TR - R - rho0);
                if constexpr (R % 4 == 0) {
#pragma unroll
                    for (int q = 0; q < R / 4; ++q) {
                        const float4 w = *reinterpret_cast<const float4 *>(gp + 4 * q);
                        ur[R - 1 - 4 * q] = w.x;
                        ur[R - 2 - 4 * q] = w.y;
                        ur[R - 3 - 4 * q] = w.z;
                        ur[R - 4 - 4 * q] = w.w;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < R / 2; ++q) {
                        const float2 w = *reinterpret_cast<const float2 *>(gp + 2 * q);
                        ur[R - 1 - 2 * q] = w.x;
                        ur[R - 2 - 2 * q] = w.y;
                    }
                }
                if (p.decay_log1p) {
#pragma unroll
                    for (int r = 0; r < R; ++r) ur[r] = log1pf(ur[r]);
                }
            }

            // per element: A, gy, cP, cQ (and the dL/dlambda factor) for phase B,
            // held as pairs of neighbouring channels for packed fp32x2 work
            float2 A[R][V2], Gy[R][V2], P[R][V2], Q[R][V2];
            [[maybe_unused]] float2 Ed[kDec ? R : 1][V2];
            float2 IA[V2], IB[V2];             // the fold of the thread's rows, per channel pair
#pragma unroll
            for (int i = 0; i < V2; ++i) {
                IA[i] = make_float2(1.f, 1.f);
                IB[i] = make_float2(0.f, 0.f);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int64_t t = top - r;
                const bool ok = dvalid && t < p.T;
                float xk[V], xh[V], xg[V], xf[V];
                unpack(*reinterpret_cast<const Vec *>(t0 - r * TC), xk);
                unpack(*reinterpret_cast<const Vec *>(t1 - r * TC), xh);
                unpack(*reinterpret_cast<const Vec *>(tg - r * TC), xg);
                unpack(*reinterpret_cast<const Vec *>(tf - r * TC), xf);
                if (t == 0) {
#pragma unroll
                    for (int v = 0; v < V; ++v) xf[v] = h0v[v];
                }
                [[maybe_unused]] float u = 0.f;
                if constexpr (kDec) u = ur[r];
#pragma unroll
                for (int i = 0; i < V2; ++i) {
                    const float2 k2 = make_float2(xk[2 * i], xk[2 * i + 1]);
                    const float2 h2 = make_float2(xh[2 * i], xh[2 * i + 1]);
                    const float2 f2 = make_float2(xf[2 * i], xf[2 * i + 1]);
                    float2 a, cp, cq;
                    if constexpr (kDec) {
                        // the two gates' exponents in one packed multiply
                        const float2 ge = __fmul2_rn(make_float2(lam2[2 * i], lam2[2 * i + 1]), make_float2(u, u));
                        const float2 gam = make_float2(fast_exp2(ge.x), fast_exp2(ge.y));
                        BOp::coeffs_gated2(k2, h2, f2, gam, a, cp, cq);
                        // dL/dlambda gains delta A h_{t-1} (-u) = (A delta) (-u h_{t-1}):
                        // the second factor here, the first in phase B
                        const float2 e = __fmul2_rn(f2, make_float2(-u, -u));
                        Ed[r][i] = ok ? e : make_float2(0.f, 0.f);
                    } else {
                        BOp::coeffs2(k2, h2, f2, a, cp, cq);
                    }
                    // rows past T, channels past D: the identity pair
                    a = ok ? a : make_float2(1.f, 1.f);
                    const float2 gv = ok ? make_float2(xg[2 * i], xg[2 * i + 1]) : make_float2(0.f, 0.f);
                    A[r][i] = a;
                    Gy[r][i] = gv;
                    P[r][i] = cp;
                    Q[r][i] = cq;
                    // (IA, IB) <- (IA a, IB a + a gy)
                    IB[i] = __ffma2_rn(IB[i], a, __fmul2_rn(a, gv));
                    IA[i] = __fmul2_rn(IA[i], a);
                }
            }
            float2 incl[V];
#pragma unroll
            for (int i = 0; i < V2; ++i) {
                incl[2 * i] = make_float2(IA[i].x, IB[i].x);
                incl[2 * i + 1] = make_float2(IA[i].y, IB[i].y);
            }
            // scan across the J row groups of the warp
#pragma unroll
            for (int off = 1; off < J; off <<= 1) {
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    float2 o;
                    o.x = __shfl_up_sync(0xffffffffu, incl[v].x, off * CG);
                    o.y = __shfl_up_sync(0xffffffffu, incl[v].y, off * CG);
                    if (j >= off) incl[v] = Op::combine(o, incl[v]);
                }
            }
            float2 ex[V];          // the thread's exclusive prefix within its warp
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float2 o;
                o.x = __shfl_up_sync(0xffffffffu, incl[v].x, CG);
                o.y = __shfl_up_sync(0xffffffffu, incl[v].y, CG);
                ex[v] = (J > 1 && j > 0) ? o : Op::identity();
            }
            if (j == J - 1) {
#pragma unroll
                for (int v = 0; v < V; ++v) s_tot[BUF][warp][g * V + v] = incl[v];
            }
            // The warp is done with the slot and has written its summary; the
            // last of the W warps refills the slot and, for fp32 I/O, folds
            // the warp summaries and publishes the chunk summary.
            __threadfence_block();
            __syncwarp();
            unsigned int seen = 0;
            if (lane == 0) seen = atomicAdd(&s_cnt[n % S], 1u);
            seen = __shfl_sync(0xffffffffu, seen, 0);
            if (seen == W - 1) {
                __threadfence_block();
                if (lane == 0) {
                    s_cnt[n % S] = 0;
                    if (n + S < n_local) {
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        issue_tile(n + S);
                    }
                }
                if constexpr (kFoldInData) {
                    const int ch = lane * CV;
                    float2 total[CV];
                    fold_warps<Op, CV, TC, W>(s_tot[BUF], ch, total);
#pragma unroll
                    for (int v = 0; v < CV; ++v) s_total[BUF][ch + v] = total[v];
                    const bool publish =
                        (p.n_chunks > 1) && (int64_t(tc.c) < p.n_chunks - 1) && (tile != p.drop_tile);
                    if (publish && tc.c > 0) publish_summary<CV, TC>(p, tile, ch, total);
                }
            }
            named_barrier_arrive(1 + BUF, NT);

            // ---- phase B: replay lam from the thread's incoming gradient
            named_barrier_sync(3 + BUF, NT);
            float2 lam[V2];
            [[maybe_unused]] float2 dl2[V2];
#pragma unroll
            for (int i = 0; i < V2; ++i) {
                const int c0 = g * V + 2 * i;
                lam[i] = make_float2(Op::apply(ex[2 * i], Op::apply(s_tot[BUF][warp][c0], s_hin[BUF][c0])),
                                     Op::apply(ex[2 * i + 1], Op::apply(s_tot[BUF][warp][c0 + 1], s_hin[BUF][c0 + 1])));
                if constexpr (kDec) dl2[i] = make_float2(0.f, 0.f);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float y0[V], y1[V];
#pragma unroll
                for (int i = 0; i < V2; ++i) {
                    const float2 delta = __fadd2_rn(Gy[r][i], lam[i]);
                    const float2 a0 = __fmul2_rn(delta, P[r][i]);
                    const float2 a1 = __fmul2_rn(delta, Q[r][i]);
                    y0[2 * i] = a0.x;
                    y0[2 * i + 1] = a0.y;
                    y1[2 * i] = a1.x;
                    y1[2 * i + 1] = a1.y;
                    lam[i] = __fmul2_rn(A[r][i], delta);
                    if constexpr (kDec) dl2[i] = __ffma2_rn(lam[i], Ed[r][i], dl2[i]);
                }
                const int64_t t = top - r;
                if (dvalid && t < p.T) {
                    Access<IO, V>::store(out0 + base + t * p.D, y0);
                    Access<IO, V>::store(out1 + base + t * p.D, y1);
                }
            }
            [[maybe_unused]] float dl[V];
            if constexpr (kDec) {
#pragma unroll
                for (int i = 0; i < V2; ++i) {
                    dl[2 * i] = dl2[i].x;
                    dl[2 * i + 1] = dl2[i].y;
                }
            }
            if constexpr (kDec) {
                // dL/dlambda: sum the warp's row groups, add the sums to the
                // tile's in shared memory; the last warp through adds the
                // tile's sums to the global ones (one atomic per channel and
                // tile) and clears them.  The next tile with this buffer
                // reaches phase B only after that warp has passed the next
                // summary barrier, so the clearing is ordered before it.
                if (bp.dlam) {
#pragma unroll
                    for (int off = CG; off < 32; off <<= 1) {
#pragma unroll
                        for (int v = 0; v < V; ++v) dl[v] += __shfl_xor_sync(0xffffffffu, dl[v], off);
                    }
                    if (j == 0) {
#pragma unroll
                        for (int v = 0; v < V; ++v) atomicAdd(&s_dl[BUF][g * V + v], dl[v]);
                    }
                    __threadfence_block();
                    __syncwarp();
                    unsigned int done = 0;
                    if (lane == 0) done = atomicAdd(&s_dcnt[BUF], 1u);
                    done = __shfl_sync(0xffffffffu, done, 0);
                    if (done == W - 1) {
                        __threadfence_block();
                        const int64_t dt0 = int64_t(tc.dt) * TC;
#pragma unroll
                        for (int v = 0; v < CV; ++v) {
                            const int ch = lane + 32 * v;
                            const float s = s_dl[BUF][ch];
                            s_dl[BUF][ch] = 0.f;
                            if (dt0 + ch < p.D) atomicAdd(bp.dlam + dt0 + ch, s);
                        }
                        if (lane == 0) s_dcnt[BUF] = 0;
                    }
                }
            }
            // the thread holding time row 0 ends with dL/d (initial state)
            if (bp.dinit && dvalid && top - (R - 1) == 0) {
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const float y[1] = {(v & 1) ? lam[v / 2].y : lam[v / 2].x};
                    Access<IO, 1>::store(static_cast<IO *>(bp.dinit) + int64_t(tc.b) * bp.dinit_bs + d0 + v, y);
                }
            }
        }
    } else {
        // ============================================== carry warp
        // The forward kernel's: per tile, resolve the incoming gradient from
        // the look-back window (issued when the previous tile was done) while
        // the data warps are in phase A; wait for the tile's warp summaries;
        // (bf16 I/O: fold them and publish the chunk summary;) write the
        // incoming gradient, release the data warps, publish the chunk's
        // final state and issue the next tile's look-back loads.  Chunk 0 in
        // processing order (the last time chunk) starts from a zero gradient
        // (the scan's initial state is null here).
        const int ch = lane * CV;
        constexpr int KW = window_long<CV>();
        LookWindow<CV, TC, KW> win;
        float init[CV];
        auto prefetch = [&](int n) {
            const TileCoord tc = tile_coord(p, uint32_t(first + int64_t(n) * G));
            if (tc.c == 0) {
#pragma unroll
                for (int v = 0; v < CV; ++v) init[v] = Op::default_init();
            } else {
                load_window<CV, TC, KW>(p, int64_t(tc.c) - 1, tc.chain, ch, win);
            }
        };
        if (n_local > 0) prefetch(0);
        for (int n = 0; n < n_local; ++n) {
            const int PB = n & 1;
            const int64_t tile = first + int64_t(n) * G;
            const TileCoord tc = tile_coord(p, uint32_t(tile));
            const int64_t c = tc.c;
            const int64_t dl = int64_t(tc.dt) * TC + ch;
            const bool publish = (p.n_chunks > 1) && (c < p.n_chunks - 1) && (tile != p.drop_tile);
            float hin[CV];
            float2 M[CV];
            int64_t q = c - 1;
            bool resolved = true;
            if (c == 0) {
#pragma unroll
                for (int v = 0; v < CV; ++v) hin[v] = init[v];
            } else if constexpr (kFoldInData) {
                look_back_from<Op, IO, CV, TC, KW>(p, c, tc.chain, tc.b, dl, ch, win, hin);
            } else {
                // walk only the window already loaded before the summary is
                // published (the next chunk's look-back may wait for it)
#pragma unroll
                for (int v = 0; v < CV; ++v) M[v] = Op::identity();
                int consumed;
                resolved = resolve_window<Op, IO, CV, TC, KW>(p, q, win, tc.b, dl, M, hin, consumed);
                q -= consumed;
            }
            named_barrier_sync(1 + PB, NT);
            if constexpr (!kFoldInData) {
                float2 total[CV];
                fold_warps<Op, CV, TC, W>(s_tot[PB], ch, total);
#pragma unroll
                for (int v = 0; v < CV; ++v) s_total[PB][ch + v] = total[v];
                if (publish && c > 0) publish_summary<CV, TC>(p, tile, ch, total);
                if (!resolved) {
                    load_window<CV, TC, KW>(p, q, tc.chain, ch, win);
                    look_back_continue<Op, IO, CV, TC, KW>(p, q, tc.chain, tc.b, dl, ch, win, M, hin);
                }
            }
#pragma unroll
            for (int v = 0; v < CV; ++v) s_hin[PB][ch + v] = hin[v];
            named_barrier_arrive(3 + PB, NT);
            if (publish) {
                float fin[CV];
#pragma unroll
                for (int v = 0; v < CV; ++v) fin[v] = Op::apply(s_total[PB][ch + v], hin[v]);
                publish_state<CV, TC>(p, tile, ch, fin);
            }
            if (n + 1 < n_local) prefetch(n + 1);
        }
    }
}

}  // namespace sgr
