// scan_backward.cuh -- gradients of the two scans (reverse-time scans).
//
// For a loss L with upstream gradient gy_t = dL/d out_t on every output row,
// the gradient flowing back into the state is itself a linear recurrence,
// run from the last step to the first.  With lam the gradient reaching out_t
// from the steps after t (0 after the last step):
//   delta_t = gy_t + lam                      (total dL/d out_t)
//   d in0_t = delta_t cP_t,  d in1_t = delta_t cQ_t  (cP, cQ: local partials)
//   lam     = A_t delta_t,   A_t = d out_t / d (state before step t)
// and after step 0, lam is dL/d (initial state).  Written as
// lam <- A_t lam + A_t gy_t it is the affine pair (A_t, A_t gy_t) composed in
// reverse time, so the forward engine's affine operator, chunk hand-off and
// look-back carry it unchanged: the tile kernel below numbers chunks in
// processing order (processing chunk c covers time chunk n_chunks - 1 - c)
// and a thread walks its rows from the highest time index down.
//
// Local partials (page "Mingru Pytorch": the minGRU layer is a trainable
// module; page "MinMax Recurrent Neural Cascades", Key properties: training
// with bounded gradients; the pages print no derivative, these are the chain
// rule through the recurrences):
//   minGRU  out = (1 - z) h + z g(hx), z = sigmoid(k):
//           A = 1 - z,  cP = z (1 - z) (g(hx) - h),  cQ = z g'(hx),
//           g'(x) = 1 for x >= 0, sigmoid(x) sigmoid(-x) otherwise;
//   MinMax  out = max(m, s), m = min(r, x): equal operands of min / max share
//           the gradient evenly (PyTorch's elementwise minimum / maximum):
//           A = dout/dm dm/dx,  cP = dout/dm dm/dr,  cQ = dout/ds.
#pragma once

#include "scan_engine.cuh"

namespace sgr {

struct MinGRUBwd {
    static constexpr bool kDecay = false;
    // (k, hx, state before the step) -> (A, cP, cQ); the same exp2 / shared
    // reciprocal evaluation of sigmoid(+-|x|) as the forward activations
    static __device__ __forceinline__ void coeffs(float k, float hx, float h, float &A, float &cP,
                                                  float &cQ) {
        coeffs_gated(k, hx, h, 1.f, A, cP, cQ);
    }
    // with the state entering the step gated by gamma (time decay):
    // out = (1 - z) gamma h + z g, so A = (1 - z) gamma and cP = z (1 - z) (g - gamma h)
    static __device__ __forceinline__ void coeffs_gated(float k, float hx, float h, float gamma,
                                                        float &A, float &cP, float &cQ) {
        const float ek = fast_exp2(fabsf(k) * kNegLog2e);
        const float eh = fast_exp2(fabsf(hx) * kNegLog2e);
        const float dk = 1.f + ek, dh = 1.f + eh;
        const float inv = fast_rcp(dk * dh);
        const float rk = dh * inv;          // sigmoid(|k|)
        const float rh = dk * inv;          // sigmoid(|hx|)
        const float sk = ek * rk;           // sigmoid(-|k|)
        const float sh = eh * rh;           // sigmoid(-|hx|)
        const bool kpos = k >= 0.f;
        const float z = kpos ? rk : sk;
        A = (kpos ? sk : rk) * gamma;
        const bool hpos = hx >= 0.f;
        const float g = hpos ? hx + 0.5f : sh;
        const float gp = hpos ? 1.f : sh * rh;
        cP = (sk * rk) * (g - gamma * h);
        cQ = z * gp;
    }
    // the same for two elements, the arithmetic in packed fp32x2 operations
    // (the MUFU operations and the sign selects stay per element)
    static __device__ __forceinline__ void coeffs_gated2(float2 k, float2 hx, float2 h, float2 gamma,
                                                         float2 &A, float2 &cP, float2 &cQ) {
        const float2 c = make_float2(kNegLog2e, kNegLog2e), one = make_float2(1.f, 1.f);
        const float2 tk = __fmul2_rn(make_float2(fabsf(k.x), fabsf(k.y)), c);
        const float2 th = __fmul2_rn(make_float2(fabsf(hx.x), fabsf(hx.y)), c);
        const float2 ek = make_float2(fast_exp2(tk.x), fast_exp2(tk.y));
        const float2 eh = make_float2(fast_exp2(th.x), fast_exp2(th.y));
        const float2 dk = __fadd2_rn(ek, one), dh = __fadd2_rn(eh, one);
        const float2 pr = __fmul2_rn(dk, dh);
        const float2 inv = make_float2(fast_rcp(pr.x), fast_rcp(pr.y));
        const float2 rk = __fmul2_rn(dh, inv);           // sigmoid(|k|)
        const float2 rh = __fmul2_rn(dk, inv);           // sigmoid(|hx|)
        const float2 sk = __fmul2_rn(ek, rk);            // sigmoid(-|k|)
        const float2 sh = __fmul2_rn(eh, rh);            // sigmoid(-|hx|)
        const bool kp0 = k.x >= 0.f, kp1 = k.y >= 0.f;
        const bool hp0 = hx.x >= 0.f, hp1 = hx.y >= 0.f;
        const float2 z = make_float2(kp0 ? rk.x : sk.x, kp1 ? rk.y : sk.y);
        A = __fmul2_rn(make_float2(kp0 ? sk.x : rk.x, kp1 ? sk.y : rk.y), gamma);
        const float2 hp = __fadd2_rn(hx, make_float2(0.5f, 0.5f));
        const float2 shrh = __fmul2_rn(sh, rh);
        const float2 g = make_float2(hp0 ? hp.x : sh.x, hp1 ? hp.y : sh.y);
        const float2 gp = make_float2(hp0 ? 1.f : shrh.x, hp1 ? 1.f : shrh.y);
        const float2 gmh = __ffma2_rn(make_float2(-gamma.x, -gamma.y), h, g);    // g - gamma h
        cP = __fmul2_rn(__fmul2_rn(sk, rk), gmh);
        cQ = __fmul2_rn(z, gp);
    }
    static __device__ __forceinline__ void coeffs2(float2 k, float2 hx, float2 h, float2 &A, float2 &cP,
                                                   float2 &cQ) {
        coeffs_gated2(k, hx, h, make_float2(1.f, 1.f), A, cP, cQ);
    }
    static __device__ __forceinline__ float default_state() { return 0.f; }
};

struct MinGRUDecayBwd : MinGRUBwd {
    static constexpr bool kDecay = true;
};

struct MinMaxBwd {
    static constexpr bool kDecay = false;
    static __device__ __forceinline__ void coeffs(float r, float s, float x, float &A, float &cP,
                                                  float &cQ) {
        const float m = fminf(r, x);
        const float dm_dr = r < x ? 1.f : (r == x ? 0.5f : 0.f);
        const float dout_dm = m > s ? 1.f : (m == s ? 0.5f : 0.f);
        A = dout_dm * (1.f - dm_dr);
        cP = dout_dm * dm_dr;
        cQ = 1.f - dout_dm;
    }
    static __device__ __forceinline__ void coeffs2(float2 r, float2 s, float2 x, float2 &A, float2 &cP,
                                                   float2 &cQ) {
        coeffs(r.x, s.x, x.x, A.x, cP.x, cQ.x);
        coeffs(r.y, s.y, x.y, A.y, cP.y, cQ.y);
    }
    static __device__ __forceinline__ float default_state() { return 0.f; }
};

struct BwdParams {
    ScanParams s;         // in0, in1, out = d in0, hand-off words; s.init is null
                          // (the reverse scan starts from a zero gradient)
    const void *fwd;      // forward output (B, T, D): the state before step t is fwd[t-1]
    const void *gy;       // dL/d out (B, T, D)
    const void *init;     // forward initial state rows (B, D) or null (zero state)
    int64_t init_bs;
    void *out1;           // d in1 (B, T, D)
    void *dinit;          // dL/d initial state (B, D) rows or null
    int64_t dinit_bs;
    float *dlam;          // time decay: dL/d lambda (D,), accumulated (zeroed by the host), or null
};

// One block per tile, W data warps + 1 carry warp, the tile kernel's lane
// layout (lane (g, j) of warp w owns channels [g V, g V + V) of processing rows
// [(w J + j) R, (w J + j) R + R)); processing row rho of a tile is time row
// ct TR + TR - 1 - rho.  Tiles are numbered chain-fastest in processing order
// and, when the sequence spans several chunks, handed to persistent blocks by
// a ticket counter (for_each_ticket), so every look-back waits on a tile that
// a running block holds.  It runs the gradients the copy-engine-fed kernels
// do not take: unaligned rows and shapes with under two tiles per SM (aligned
// narrow batches take scan_pipelined_backward.cuh, wide ones the
// channel-sequential gradient).
template <class BOp, typename IO, int V, int CG, int R, int W, int MINB>
__global__ void __launch_bounds__((W + 1) * 32, MINB) scan_backward_kernel(const BwdParams bp) {
    constexpr int J = 32 / CG;
    constexpr int TR = W * J * R;
    constexpr int TC = CG * V;
    constexpr int CV = TC / 32;
    constexpr uint32_t NT = (W + 1) * 32;
    static_assert(CG * J == 32 && TC % 32 == 0, "lane layout");
    using Op = MinGRUOp;              // affine pairs carry the gradient

    __shared__ float2 s_tot[W][TC];

    const ScanParams &p = bp.s;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    for_each_ticket(p.ticket, p.n_tiles, [&](const int64_t tile, auto take_next) {

    if (warp < W) {
        const TileCoord tc = tile_coord(p, uint32_t(tile));
        const int64_t ct = p.n_chunks - 1 - int64_t(tc.c);     // time chunk
        const int g = lane % CG;
        const int j = lane / CG;
        const int64_t d0 = int64_t(tc.dt) * TC + int64_t(g) * V;
        const bool dvalid = d0 < p.D;
        const int64_t top = ct * TR + TR - 1 - int64_t(warp * J + j) * R;   // time row of r = 0
        const int64_t base = (int64_t(tc.b) * p.T) * p.D + d0;
        const IO *in0 = static_cast<const IO *>(p.in0);
        const IO *in1 = static_cast<const IO *>(p.in1);
        const IO *fwd = static_cast<const IO *>(bp.fwd);
        const IO *gy = static_cast<const IO *>(bp.gy);

        // rows r = 0..R-1 at time top - r: A, the upstream gradient, cP, cQ
        // (time decay: and E = (1 - z) h_{t-1} dgamma/dlambda, for dL/dlambda)
        float A[R][V], G[R][V], P[R][V], Q[R][V];
        [[maybe_unused]] float E[BOp::kDecay ? R : 1][V];
        [[maybe_unused]] float lam2[V];
        if constexpr (BOp::kDecay) {
#pragma unroll
            for (int v = 0; v < V; ++v) lam2[v] = decay_lam2(p, d0 + v);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t t = top - r;
            if (dvalid && t < p.T) {
                Access<IO, V>::load(in0 + base + t * p.D, A[r]);
                Access<IO, V>::load(in1 + base + t * p.D, P[r]);
                Access<IO, V>::load(gy + base + t * p.D, G[r]);
                if (t > 0) {
                    Access<IO, V>::load(fwd + base + (t - 1) * p.D, Q[r]);
                } else {
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        Q[r][v] = bp.init ? load_scalar<IO>(static_cast<const IO *>(bp.init) +
                                                            int64_t(tc.b) * bp.init_bs + d0 + v)
                                          : BOp::default_state();
                    }
                }
            } else {
#pragma unroll
                for (int v = 0; v < V; ++v) { A[r][v] = 0.f; P[r][v] = 0.f; G[r][v] = 0.f; Q[r][v] = 0.f; }
            }
        }
        float2 incl[V];
#pragma unroll
        for (int v = 0; v < V; ++v) incl[v] = Op::identity();
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const bool ok = dvalid && (top - r) < p.T;
            [[maybe_unused]] float u = 0.f;
            if constexpr (BOp::kDecay) {
                if ((top - r) < p.T) u = decay_u(p, tc.b, top - r);
            }
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float a, cp, cq;
                if constexpr (BOp::kDecay) {
                    const float gamma = decay_gamma(lam2[v], u);
                    BOp::coeffs_gated(A[r][v], P[r][v], Q[r][v], gamma, a, cp, cq);
                    // dL/dlambda gains delta (1 - z) h_{t-1} dgamma/dlambda
                    //   = delta A h_{t-1} (-u)   (dgamma/dlambda = -u gamma; 0 where gamma is 0)
                    E[r][v] = -u * a * Q[r][v];
                } else {
                    BOp::coeffs(A[r][v], P[r][v], Q[r][v], a, cp, cq);
                }
                a = ok ? a : 1.f;                 // rows past T: identity pair, gy = 0
                A[r][v] = a;
                P[r][v] = cp;
                Q[r][v] = cq;
                incl[v] = Op::combine(incl[v], make_float2(a, a * G[r][v]));
            }
        }
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
        if (j == J - 1) {
#pragma unroll
            for (int v = 0; v < V; ++v) s_tot[warp][g * V + v] = incl[v];
        }
        float2 excl[V];
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float2 o;
            o.x = __shfl_up_sync(0xffffffffu, incl[v].x, CG);
            o.y = __shfl_up_sync(0xffffffffu, incl[v].y, CG);
            excl[v] = (J > 1 && j > 0) ? o : Op::identity();
        }
        named_barrier_sync(1, NT);   // summaries are in shared memory
        named_barrier_sync(2, NT);   // the carry warp has written the incoming gradients
        take_next();                 // the tile's look-back is over: take the next ticket

        float lam[V], dl[V];
#pragma unroll
        for (int v = 0; v < V; ++v) {
            lam[v] = Op::apply(excl[v], s_tot[warp][g * V + v].x);
            dl[v] = 0.f;
        }
        IO *out0 = static_cast<IO *>(p.out);
        IO *out1 = static_cast<IO *>(bp.out1);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float y0[V], y1[V];
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const float delta = G[r][v] + lam[v];
                y0[v] = delta * P[r][v];
                y1[v] = delta * Q[r][v];
                if constexpr (BOp::kDecay) dl[v] = fmaf(delta, E[r][v], dl[v]);
                lam[v] = A[r][v] * delta;
            }
            const int64_t t = top - r;
            if (dvalid && t < p.T) {
                Access<IO, V>::store(out0 + base + t * p.D, y0);
                Access<IO, V>::store(out1 + base + t * p.D, y1);
            }
        }
        if constexpr (BOp::kDecay) {
            // dL/dlambda: sum the warp's row groups, one atomic add per channel and warp
            if (bp.dlam) {
#pragma unroll
                for (int off = CG; off < 32; off <<= 1) {
#pragma unroll
                    for (int v = 0; v < V; ++v) dl[v] += __shfl_xor_sync(0xffffffffu, dl[v], off);
                }
                if (j == 0 && dvalid) {
#pragma unroll
                    for (int v = 0; v < V; ++v) atomicAdd(bp.dlam + d0 + v, dl[v]);
                }
            }
        }
        // the thread holding time row 0 ends with dL/d (initial state)
        if (bp.dinit && dvalid && top - (R - 1) == 0) {
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const float y[1] = {lam[v]};
                Access<IO, 1>::store(static_cast<IO *>(bp.dinit) + int64_t(tc.b) * bp.dinit_bs + d0 + v, y);
            }
        }
    } else {
        named_barrier_sync(1, NT);
        carry_tile<Op, IO, CV, TC, W>(p, tile, s_tot, lane, [&] { named_barrier_sync(2, NT); });
    }
    });
}

}  // namespace sgr
