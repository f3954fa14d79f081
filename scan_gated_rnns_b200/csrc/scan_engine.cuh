// scan_engine.cuh -- single-pass chunked scan engine for element-wise
// recurrences over the time axis of a (B, T, D) tensor, for sm_100a.
//
// Both recurrences the library serves are compositions of per-step maps
// f_t acting on one channel's state:
//   minGRU (page "Mingru Pytorch", log-space minGRU):  f_t(h) = a_t h + b_t,
//       a_t = 1 - z_t = sigmoid(-k_t),  b_t = z_t g(hx_t);
//   MinMax neuron (page "MinMax Recurrent Neural Cascades", The model, item 3):
//       f_t(x) = max(min(x, u_t), l_t),  u_t = r_t, l_t = s_t.
// Each family is closed under composition, so a run of steps is summarised by
// one pair and summaries compose associatively -- this is what gives the scan
// its O(log T)-depth parallel form (page "MinMax Recurrent Neural Cascades",
// Key properties: parallel training):
//   affine: (A1, B1) then (A2, B2) = (A1 A2, B1 A2 + B2)
//   clamp : (U1, L1) then (U2, L2) = (min(U1, U2), max(min(L1, U2), L2))
// (the clamp rule is min distributing over max, exact in a total order).
// The minGRU log-space formula h = exp(a* + logcumsumexp(log z + log g - a*))
// is the closed form of the same affine composition; evaluating the pairs in
// linear space gives that function with fp32 errors relative to each term
// (no cancellation: all terms are positive) and with 3-4 MUFU ops per
// element instead of about 9 for the log-space pairs (MinGRULogOp below,
// kept as the measured alternative).
//
// Work decomposition (one thread block = one tile of TR rows x TC channels):
//   load   : each thread loads R consecutive rows x V channels of both inputs
//            with 128-bit streaming loads (D fastest => a warp reads whole
//            128-byte row segments), all issued before any is consumed;
//   phase 1: activations fused in registers, then a sequential fold of the
//            thread's R steps into one pair per channel;
//   phase 2: exclusive scan of the sub-chunk pairs: shuffles across the J
//            row-groups of a warp, shared memory across the W warps;
//   carry  : the tile's incoming state -- the initial state for the first
//            chunk, otherwise decoupled look-back over the summaries the
//            earlier chunks of the same channels publish in the workspace;
//   phase 3: each thread replays its R steps sequentially from its incoming
//            state (one FMA per element for minGRU) and streams the outputs.
// Inputs are read from HBM once and outputs written once: the algorithmic
// 3 x elem_bytes per element (plus the initial state) is the whole traffic
// apart from the workspace, which is a few bytes per tile and channel and
// stays in L2.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda.h>
#include <stdint.h>

#include <type_traits>

namespace sgr {

// --------------------------------------------------- hardware approximations
//
// exp(x) = 2^(x log2 e) with the MUFU's 2^x and 1/x approximations (ftz:
// results below the normal range flush to 0, which only ever replaces a gate
// below 1e-38 by 0).
constexpr float kNegLog2e = -1.4426950408889634f;
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float fast_rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// log2(x) by the MUFU approximation (x <= 0 gives -inf / NaN)
__device__ __forceinline__ float fast_lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------------- operators

struct MinGRUOp {
    static constexpr bool kDecay = false;
    // pair (A, B): state -> A * state + B
    static __device__ __forceinline__ float2 identity() { return make_float2(1.f, 0.f); }
    // (first, then) -> composition
    static __device__ __forceinline__ float2 combine(float2 p, float2 q) {
        return make_float2(p.x * q.x, fmaf(p.y, q.x, q.y));
    }
    static __device__ __forceinline__ float apply(float2 p, float x) { return fmaf(p.x, x, p.y); }
    // input values that produce the identity pair (padding rows): k = -inf gives
    // z = 0 exactly, so a = 1 and b = 0 * g(0) = 0
    static __device__ __forceinline__ float pad0() { return -INFINITY; }
    static __device__ __forceinline__ float pad1() { return 0.f; }
    // fused activations: (k, hx) -> (a, b) = (sigmoid(-k), sigmoid(k) * g(hx)).
    // With e = exp(-|x|) in [0, 1]: sigmoid(-|x|) = e/(1+e) =: s <= 1/2 and
    // sigmoid(|x|) = 1 - s (no cancellation since s <= 1/2; exactly 1 - 0 = 1
    // when e underflows, so k = -inf gives a = 1 and k = +inf gives z = 1).
    // The two reciprocals 1/(1+ek), 1/(1+eh) share one division:
    // inv = 1/((1+ek)(1+eh)).  MUFU work: 2 exp2 + 1 reciprocal (hardware
    // approximations, relative error ~2^-22), the rest in packed fp32x2 pairs.
    static __device__ __forceinline__ void element(float k, float hx, float &a, float &b) {
        const float2 e = make_float2(fast_exp2(fabsf(k) * kNegLog2e), fast_exp2(fabsf(hx) * kNegLog2e));
        const float2 d = __fadd2_rn(e, make_float2(1.f, 1.f));               // (1+ek, 1+eh)
        const float inv = fast_rcp(d.x * d.y);
        const float2 rr = __fmul2_rn(make_float2(d.y, d.x), make_float2(inv, inv));  // (1/(1+ek), 1/(1+eh))
        const float2 sg = __fmul2_rn(e, rr);     // (sigmoid(-|k|), sigmoid(-|hx|))
        const float kbig = 1.f - sg.x;          // sigmoid(|k|)
        const bool kpos = k >= 0.f;
        const float z = kpos ? kbig : sg.x;
        a = kpos ? sg.x : kbig;
        const float g = (hx >= 0.f) ? hx + 0.5f : sg.y;
        b = z * g;
    }
    // The pairs of two steps (rows) of one channel, each fp32x2 operation
    // packed across the two steps (two independent dependency chains per
    // instruction stream), for the kernels where one lane owns one channel.
    // Evaluated without the sign selects of element(): with e = 2^(k log2 e),
    //   a = sigmoid(-k) = 1 / (1 + e),  z = sigmoid(k) = e a,
    // both relative-accurate for either sign of k (a product and a quotient
    // of correctly signed positive terms, no cancellation).  k log2 e is
    // clamped at 126 so that e stays finite: beyond k ~ 87 that leaves
    // a = 2^-126 (instead of a smaller positive number) and z = 1, and
    // k = +inf gives z = 1 exactly, k = -inf gives e = 0, a = 1, z = 0.
    // g(hx) = max(hx + 0.5, sigmoid(hx)) with sigmoid(hx) = 1 / (1 + 2^(-hx
    // log2 e)) holds for every hx (hx + 0.5 - sigmoid(hx) is increasing and
    // 0 at hx = 0); hx = -inf gives 0, large hx gives hx + 0.5.  MUFU work:
    // 2 exp2 + 2 reciprocals per element, about 5 instructions fewer than
    // element().
    static __device__ __forceinline__ void element_rows(float k0, float hx0, float k1, float hx1, float2 &a,
                                                        float2 &b) {
        const float2 tk = __fmul2_rn(make_float2(k0, k1), make_float2(-kNegLog2e, -kNegLog2e));
        const float2 th = __fmul2_rn(make_float2(hx0, hx1), make_float2(kNegLog2e, kNegLog2e));
        const float2 one = make_float2(1.f, 1.f);
        const float2 ek = make_float2(fast_exp2(fminf(tk.x, 126.f)), fast_exp2(fminf(tk.y, 126.f)));
        const float2 dk = __fadd2_rn(ek, one);                                  // 1 + e^k
        const float2 dh = __fadd2_rn(make_float2(fast_exp2(th.x), fast_exp2(th.y)), one);   // 1 + e^-hx
        a = make_float2(fast_rcp(dk.x), fast_rcp(dk.y));                         // sigmoid(-k)
        const float2 z = __fmul2_rn(ek, a);                                     // sigmoid(k)
        const float2 s = make_float2(fast_rcp(dh.x), fast_rcp(dh.y));            // sigmoid(hx)
        const float2 hp = __fadd2_rn(make_float2(hx0, hx1), make_float2(0.5f, 0.5f));
        b = __fmul2_rn(z, make_float2(fmaxf(hp.x, s.x), fmaxf(hp.y, s.y)));
    }
    // The same pairs with one reciprocal shared by the two gates (3 MUFU
    // operations per element instead of 4), for bf16 I/O: with
    // e_k = 2^(min(k log2 e, 120)) and e_h = 2^(-|hx| log2 e) <= 1,
    // q = 1 / ((1 + e_k)(1 + e_h)) stays a normal number (the product is at
    // most 2^121), z = e_k (1 + e_h) q = sigmoid(k), a = 1 - z,
    // sigmoid(-|hx|) = e_h (1 + e_k) q and g = max(hx + 0.5, sigmoid(-|hx|))
    // (equal to g(hx) for either sign of hx).  a = 1 - z is exact where
    // k <= 0 (z <= 1/2) and carries an absolute error of an fp32 ulp of 1
    // where k >> 0: far below the bf16 rounding of the outputs, not enough
    // for the fp32 bar on long closed-gate stretches, hence bf16 only.
    // k = -inf gives z = 0 and a = 1 exactly; hx = -inf gives g = 0.
    static __device__ __forceinline__ void element_rows_lean(float k0, float hx0, float k1, float hx1,
                                                             float2 &a, float2 &b) {
        const float2 tk = __fmul2_rn(make_float2(k0, k1), make_float2(-kNegLog2e, -kNegLog2e));
        const float2 ek = make_float2(fast_exp2(fminf(tk.x, 120.f)), fast_exp2(fminf(tk.y, 120.f)));
        const float2 eh = make_float2(fast_exp2(fabsf(hx0) * kNegLog2e), fast_exp2(fabsf(hx1) * kNegLog2e));
        const float2 one = make_float2(1.f, 1.f);
        const float2 dk = __fadd2_rn(ek, one), dh = __fadd2_rn(eh, one);
        const float2 pr = __fmul2_rn(dk, dh);
        const float2 q = make_float2(fast_rcp(pr.x), fast_rcp(pr.y));
        const float2 z = __fmul2_rn(ek, __fmul2_rn(dh, q));                    // sigmoid(k)
        a = __ffma2_rn(z, make_float2(-1.f, -1.f), one);                        // sigmoid(-k)
        const float2 sh = __fmul2_rn(eh, __fmul2_rn(dk, q));                   // sigmoid(-|hx|)
        const float2 hp = __fadd2_rn(make_float2(hx0, hx1), make_float2(0.5f, 0.5f));
        b = __fmul2_rn(z, make_float2(fmaxf(hp.x, sh.x), fmaxf(hp.y, sh.y)));
    }
    static constexpr bool kLeanRows = true;
    // fold a step into a running pair, two channels at once: (A, B) <- (A a, B a + b)
    static __device__ __forceinline__ void fold2(float2 &A, float2 &B, float2 a, float2 b) {
        B = __ffma2_rn(B, a, b);
        A = __fmul2_rn(A, a);
    }
    // replay one step for two channels: h <- a h + b
    static __device__ __forceinline__ float2 step2(float2 a, float2 b, float2 h) { return __ffma2_rn(a, h, b); }
    // one step of phase 3
    static __device__ __forceinline__ float step(float a, float b, float x) { return fmaf(a, x, b); }
    // initial state when none is given
    static __device__ __forceinline__ float default_init() { return 0.f; }
    // the carried state is the state itself (see MinGRULogOp)
    static constexpr bool kLogSpace = false;
    static __device__ __forceinline__ float state_in(float h) { return h; }
    static __device__ __forceinline__ float state_out(float s) { return s; }
};

struct MinMaxOp {
    static constexpr bool kDecay = false;
    // pair (U, L): state -> max(min(state, U), L)
    static __device__ __forceinline__ float2 identity() { return make_float2(INFINITY, -INFINITY); }
    static __device__ __forceinline__ float2 combine(float2 p, float2 q) {
        return make_float2(fminf(p.x, q.x), fmaxf(fminf(p.y, q.x), q.y));
    }
    static __device__ __forceinline__ float apply(float2 p, float x) { return fmaxf(fminf(x, p.x), p.y); }
    static __device__ __forceinline__ float pad0() { return INFINITY; }
    static __device__ __forceinline__ float pad1() { return -INFINITY; }
    static __device__ __forceinline__ void element(float r, float s, float &u, float &l) { u = r; l = s; }
    static __device__ __forceinline__ void element_rows(float r0, float s0, float r1, float s1, float2 &u,
                                                        float2 &l) {
        u = make_float2(r0, r1);
        l = make_float2(s0, s1);
    }
    static constexpr bool kLeanRows = false;
    static __device__ __forceinline__ float step(float u, float l, float x) { return fmaxf(fminf(x, u), l); }
    static __device__ __forceinline__ float default_init() { return 0.f; }
    static __device__ __forceinline__ void fold2(float2 &U, float2 &L, float2 u, float2 l) {
        L = make_float2(fmaxf(fminf(L.x, u.x), l.x), fmaxf(fminf(L.y, u.y), l.y));
        U = make_float2(fminf(U.x, u.x), fminf(U.y, u.y));
    }
    static __device__ __forceinline__ float2 step2(float2 u, float2 l, float2 x) {
        return make_float2(fmaxf(fminf(x.x, u.x), l.x), fmaxf(fminf(x.y, u.y), l.y));
    }
    static constexpr bool kLogSpace = false;
    static __device__ __forceinline__ float state_in(float h) { return h; }
    static __device__ __forceinline__ float state_out(float s) { return s; }
};

// log2(2^x + 2^y), exact at -inf: the larger term plus log2(1 + 2^-(gap));
// both -inf gives -inf (not the NaN of -inf - -inf).  2 MUFU operations.
__device__ __forceinline__ float lse2(float x, float y) {
    const float m = fmaxf(x, y);
    const float r = m + fast_lg2(1.f + fast_exp2(fminf(x, y) - m));
    return m == -INFINITY ? m : r;
}

// minGRU evaluated in log space, the form the page's layer computes (page
// "Mingru Pytorch", Requirements & limits: the log-space numerically stable
// minGRU): with log a_t = -softplus(k_t), log b_t = log z_t + log g(hx_t),
//   log h_t = logaddexp(log a_t + log h_{t-1}, log b_t),
// which unrolled is a*_t + logcumsumexp(log b_s - a*_s) with a*_t the running
// sum of log a.  A pair (LA, LB) maps a log-state x to logaddexp(LA + x, LB);
// composing two steps adds the LA and takes the logaddexp of the LB shifted by
// the later LA, so the scan engine's chunk hand-off, look-back and replay
// carry it unchanged, with the state held as log2 h (h = 0 is -inf) and
// exponentiated only at the store.  All logs are base 2 (the MUFU's): per
// element 4 MUFU operations for the activations, 2 for the fold and 3 for the
// replay and the store, against 3-4 in all for the linear pairs.  Kept as the
// measured alternative to the linear evaluation, not the default.
//   softplus2(k) = log2(1 + 2^(k log2 e)) = max(kl, 0) + log2(1 + 2^-|kl|),
//   LA = -softplus2(k),  log2 z = min(kl, 0) - log2(1 + 2^-|kl|),
//   log2 g(hx) = log2(hx + 0.5) (hx >= 0), hl - log2(1 + 2^hl) (hx < 0),
// kl = k log2 e, hl = hx log2 e.  k = -inf gives the identity (0, -inf).
struct MinGRULogOp {
    static constexpr bool kDecay = false;
    static constexpr bool kLeanRows = false;
    static constexpr bool kLogSpace = true;
    static __device__ __forceinline__ float2 identity() { return make_float2(0.f, -INFINITY); }
    static __device__ __forceinline__ float2 combine(float2 p, float2 q) {
        return make_float2(p.x + q.x, lse2(p.y + q.x, q.y));
    }
    static __device__ __forceinline__ float apply(float2 p, float x) { return lse2(p.x + x, p.y); }
    static __device__ __forceinline__ float pad0() { return -INFINITY; }
    static __device__ __forceinline__ float pad1() { return 0.f; }
    static __device__ __forceinline__ void element(float k, float hx, float &la, float &lb) {
        const float kl = k * -kNegLog2e, hl = hx * -kNegLog2e;
        const float lk = fast_lg2(1.f + fast_exp2(-fabsf(kl)));
        const bool hpos = hx >= 0.f;
        const float lg = fast_lg2(hpos ? hx + 0.5f : 1.f + fast_exp2(hl));
        la = -(fmaxf(kl, 0.f) + lk);
        lb = (fminf(kl, 0.f) - lk) + (hpos ? lg : hl - lg);
    }
    static __device__ __forceinline__ void fold2(float2 &A, float2 &B, float2 a, float2 b) {
        B = make_float2(lse2(B.x + a.x, b.x), lse2(B.y + a.y, b.y));
        A = make_float2(A.x + a.x, A.y + a.y);
    }
    static __device__ __forceinline__ float2 step2(float2 a, float2 b, float2 h) {
        return make_float2(lse2(a.x + h.x, b.x), lse2(a.y + h.y, b.y));
    }
    static __device__ __forceinline__ float step(float a, float b, float x) { return lse2(a + x, b); }
    static __device__ __forceinline__ float default_init() { return 0.f; }
    // the carried state is log2 h: taken from an initial state (h > 0; 0
    // gives -inf) and returned to h at the store
    static __device__ __forceinline__ float state_in(float h) { return fast_lg2(h); }
    static __device__ __forceinline__ float state_out(float s) { return fast_exp2(s); }
};

// minGRU with time decay (page "Your first delta model", Step 5: every mixer
// takes the decay contract; the carried state is gated once per token at the
// token boundary, before the token's own write): the state entering token t
// is gamma_t h_{t-1}, gamma_t = exp(-lambda_d u_bt), u the gap before the
// token (or log1p of it), so the per-step pair is (a_t gamma_t, b_t).  A gap
// with lambda u > 1e4 wipes the state (gamma = 0 exactly).
struct MinGRUDecayOp : MinGRUOp {
    static constexpr bool kDecay = true;
};

// The step pairs of two elements (two channels of a row in the pipelined
// kernel) in packed fp32x2 operations: bf16 I/O takes the shared-reciprocal
// form, fp32 I/O the form with relative-accurate gates for either sign; the
// log-space operator evaluates them one by one.
template <class Op, typename IO>
__device__ __forceinline__ void element_pair(float k0, float hx0, float k1, float hx1, float2 &a, float2 &b) {
    if constexpr (Op::kLogSpace) {
        Op::element(k0, hx0, a.x, b.x);
        Op::element(k1, hx1, a.y, b.y);
    } else if constexpr (sizeof(IO) == 2 && Op::kLeanRows) {
        Op::element_rows_lean(k0, hx0, k1, hx1, a, b);
    } else {
        Op::element_rows(k0, hx0, k1, hx1, a, b);
    }
}

// gamma = exp(-lambda u) = 2^(lam2 u) with lam2 = -lambda log2 e (<= 0).
// The wipe needs no compare: the MUFU 2^x flushes every result below the
// normal range to +0, so gamma is exactly 0 for all lambda u above about 87.3
// (2^-126 = e^-87.3), which includes every gap past the 1e4 clamp; the
// gradients then see gamma = 0 and dgamma/dlambda = -u gamma = 0 there too.
__device__ __forceinline__ float decay_gamma(float lam2, float u) { return fast_exp2(lam2 * u); }

// ------------------------------------------------------------ memory access

// V consecutive elements of type IO at p (16-byte aligned when V > 1),
// widened to fp32.  Streaming loads: every input byte is read exactly once.
template <typename IO, int V> struct Access;

template <> struct Access<float, 4> {
    static __device__ __forceinline__ void load(const float *p, float (&x)[4]) {
        const float4 t = __ldcs(reinterpret_cast<const float4 *>(p));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    }
    static __device__ __forceinline__ void store(float *p, const float (&x)[4]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
    }
};

template <> struct Access<float, 1> {
    static __device__ __forceinline__ void load(const float *p, float (&x)[1]) { x[0] = __ldcs(p); }
    static __device__ __forceinline__ void store(float *p, const float (&x)[1]) { __stcs(p, x[0]); }
};

template <> struct Access<__nv_bfloat16, 8> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&x)[8]) {
        const uint4 t = __ldcs(reinterpret_cast<const uint4 *>(p));
        const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&x)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&h);
        }
        __stcs(reinterpret_cast<uint4 *>(p), make_uint4(w[0], w[1], w[2], w[3]));
    }
};

template <> struct Access<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&x)[4]) {
        const uint2 t = __ldcs(reinterpret_cast<const uint2 *>(p));
        x[0] = __uint_as_float(t.x << 16);
        x[1] = __uint_as_float(t.x & 0xffff0000u);
        x[2] = __uint_as_float(t.y << 16);
        x[3] = __uint_as_float(t.y & 0xffff0000u);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&x)[4]) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(x[0], x[1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(x[2], x[3]);
        __stcs(reinterpret_cast<uint2 *>(p),
               make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi)));
    }
};

template <> struct Access<__nv_bfloat16, 1> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&x)[1]) {
        const unsigned short u = __ldcs(reinterpret_cast<const unsigned short *>(p));
        x[0] = __uint_as_float(uint32_t(u) << 16);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&x)[1]) {
        __nv_bfloat16 h = __float2bfloat16_rn(x[0]);
        __stcs(reinterpret_cast<unsigned short *>(p), *reinterpret_cast<unsigned short *>(&h));
    }
};

// plain (coherent) scalar loads: initial states and step operands, which may
// alias a step's output
template <typename IO> __device__ __forceinline__ float load_scalar(const IO *p);
template <> __device__ __forceinline__ float load_scalar<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float load_scalar<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return __bfloat162float(*p);
}


// One vector of V elements from shared memory, widened to fp32.
template <typename IO, int V> struct VecOf;
template <> struct VecOf<float, 4> { using type = uint4; };
template <> struct VecOf<__nv_bfloat16, 4> { using type = uint2; };

__device__ __forceinline__ void unpack(const uint4 &t, float (&x)[4]) {
    x[0] = __uint_as_float(t.x); x[1] = __uint_as_float(t.y);
    x[2] = __uint_as_float(t.z); x[3] = __uint_as_float(t.w);
}
__device__ __forceinline__ void unpack(const uint2 &t, float (&x)[4]) {   // 4 x bf16
    x[0] = __uint_as_float(t.x << 16);
    x[1] = __uint_as_float(t.x & 0xffff0000u);
    x[2] = __uint_as_float(t.y << 16);
    x[3] = __uint_as_float(t.y & 0xffff0000u);
}

// ------------------------------------------------------- chunk hand-off
//
// Each chunk (tile) publishes, per channel, three 64-bit words in the
// workspace: its summary pair (A, B) and, once known, its final state S.
// Every word carries the launch epoch in its high half next to the fp32 value
// in its low half, and is written and read as one 64-bit access, so a reader
// sees either the whole current word or a stale one with another epoch.
// No flag, no fence and no second round trip is needed: a word is valid
// exactly when its epoch matches.  Layout: words[(tile * 3 + kind) * TC + ch],
// kind 0 = A, 1 = B, 2 = S.

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u64(uint64_t *p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t pack_word(uint32_t epoch, float v) {
    return (uint64_t(epoch) << 32) | uint64_t(__float_as_uint(v));
}
__device__ __forceinline__ bool word_valid(uint64_t w, uint32_t epoch) { return uint32_t(w >> 32) == epoch; }
__device__ __forceinline__ float word_value(uint64_t w) { return __uint_as_float(uint32_t(w)); }

// bounded waiting: 2^18 polls with back-off capped at 1 us => a fraction of a
// second, far above the microseconds a chunk waits for a running predecessor
constexpr uint32_t kSpinLimit = 1u << 18;
constexpr uint32_t kTimeoutBit = 1u;

// Division by a divisor fixed at launch, for values below 2^31: the
// multiply-high / add / shift form of division by invariant integers
// (Granlund and Montgomery, 1994), round-up variant.  The host picks
// s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1; then
// n / d = (umulhi(n, m) + n) >> s for every n < 2^31 (the sum fits 32 bits).
struct FastDiv {
    uint32_t d, m, s;
    __device__ __forceinline__ uint32_t div(uint32_t n) const { return (__umulhi(n, m) + n) >> s; }
};

struct ScanParams {
    const void *in0;      // k or r, (B, T, D)
    const void *in1;      // hx or s, (B, T, D)
    const void *init;     // (B, D) rows or nullptr
    int64_t init_bs;      // batch stride of init, elements
    void *out;            // (B, T, D)
    int64_t B, T, D;
    int64_t n_dt;         // channel tiles per batch row
    int64_t n_chains;     // B * n_dt
    int64_t n_chunks;     // chunks along T
    int64_t n_tiles;      // n_chains * n_chunks (< 2^31)
    FastDiv by_chains;    // tile  -> (chunk, chain)
    FastDiv by_dt;        // chain -> (b, dt)
    uint64_t *words;      // [n_tiles][3][TC] hand-off words (workspace)
    uint32_t *status;     // device status word
    uint32_t *ticket;     // chunk ticket counter, zero at launch (tile kernels), or null: tile = blockIdx.x
    uint32_t epoch;
    uint32_t spin_limit;  // polls before a chunk gives up waiting
    int64_t drop_tile;    // testing: this tile does not publish (-1: none)
    // time decay (MinGRUDecayOp only): gaps (B, T) with batch stride, rates (D,)
    const float *decay_dt;
    int64_t decay_dt_bs;
    const float *decay_lam;
    int decay_log1p;      // u = log1p(gap) instead of the gap
};

// gap before token t of batch row b, as it enters the gate
__device__ __forceinline__ float decay_u(const ScanParams &p, int64_t b, int64_t t) {
    const float g = p.decay_dt[b * p.decay_dt_bs + t];
    return p.decay_log1p ? log1pf(g) : g;
}
__device__ __forceinline__ float decay_lam2(const ScanParams &p, int64_t d) {
    return d < p.D ? -p.decay_lam[d] * 1.4426950408889634f : 0.f;
}

// Position of a tile: chunk c along T, chain = b * n_dt + dt.  All < 2^31.
struct TileCoord {
    uint32_t c, chain, b, dt;
};
__device__ __forceinline__ TileCoord tile_coord(const ScanParams &p, uint32_t tile) {
    TileCoord t;
    t.c = p.by_chains.div(tile);
    t.chain = tile - t.c * p.by_chains.d;
    t.b = p.by_dt.div(t.chain);
    t.dt = t.chain - t.b * p.by_dt.d;
    return t;
}

template <typename IO>
__device__ __forceinline__ float load_init(const ScanParams &p, int64_t b, int64_t d, float dflt) {
    if (p.init == nullptr || d >= p.D) return dflt;
    return load_scalar<IO>(static_cast<const IO *>(p.init) + b * p.init_bs + d);
}

// Publish this chunk's summary pairs for CV channels starting at ch.
template <int CV, int TC>
__device__ __forceinline__ void publish_summary(const ScanParams &p, int64_t tile, int ch,
                                                const float2 (&tot)[CV]) {
    uint64_t *w = p.words + tile * 3 * TC + ch;
#pragma unroll
    for (int v = 0; v < CV; ++v) {
        st_relaxed_u64(w + v, pack_word(p.epoch, tot[v].x));
        st_relaxed_u64(w + TC + v, pack_word(p.epoch, tot[v].y));
    }
}

template <int CV, int TC>
__device__ __forceinline__ void publish_state(const ScanParams &p, int64_t tile, int ch,
                                              const float (&st)[CV]) {
    uint64_t *w = p.words + tile * 3 * TC + 2 * TC + ch;
#pragma unroll
    for (int v = 0; v < CV; ++v) st_relaxed_u64(w + v, pack_word(p.epoch, st[v]));
}

// Decoupled look-back for CV channels of one lane: the state entering chunk c
// of `chain`.  Walks back over chunks c-1, c-2, ... reading K of them per
// round trip: a chunk whose final state S is published ends the walk; a chunk
// with only its summary (A, B) is folded in and the walk goes on; a chunk with
// neither is waited for (bounded, with back-off).  Before chunk 0 the state is
// the initial state.  Each lane works alone: its channels' words carry their
// own validity.
// chunks read per round trip: short windows for the tile kernel (few
// registers), longer ones for the pipelined kernel's carry warp
template <int CV>
constexpr int window_short() { return CV >= 4 ? 1 : (CV == 2 ? 2 : 4); }
template <int CV>
constexpr int window_long() { return CV >= 4 ? 1 : (CV == 2 ? 4 : 8); }

template <int CV, int TC, int KW>
struct LookWindow {
    static constexpr int K = KW;
    uint64_t wa[K][CV], wb[K][CV], ws[K][CV];
};

// issue the loads of the words of chunks q, q-1, ..., q-K+1
template <int CV, int TC, int KW>
__device__ __forceinline__ void load_window(const ScanParams &p, int64_t q, int64_t chain, int ch,
                                            LookWindow<CV, TC, KW> &win) {
#pragma unroll
    for (int i = 0; i < KW; ++i) {
        const int64_t qq = q - i;
        if (qq >= 0) {
            const uint64_t *w = p.words + (qq * p.n_chains + chain) * 3 * TC + ch;
#pragma unroll
            for (int v = 0; v < CV; ++v) {
                win.ws[i][v] = ld_relaxed_u64(w + 2 * TC + v);
                win.wa[i][v] = ld_relaxed_u64(w + v);
                win.wb[i][v] = ld_relaxed_u64(w + TC + v);
            }
        }
    }
}

// Walk a loaded window starting at chunk q with the running composite M.
// Returns true when the incoming state is known (hin set); otherwise the
// number of chunks folded in is in `consumed`.
template <class Op, typename IO, int CV, int TC, int KW>
__device__ __forceinline__ bool resolve_window(const ScanParams &p, int64_t q, const LookWindow<CV, TC, KW> &win,
                                               int64_t b, int64_t d_first, float2 (&M)[CV],
                                               float (&hin)[CV], int &consumed) {
    consumed = 0;
    bool done = false, stop = false;
#pragma unroll
    for (int i = 0; i < KW; ++i) {
        if (done || stop) continue;
        const int64_t qq = q - i;
        if (qq < 0) {
#pragma unroll
            for (int v = 0; v < CV; ++v)
                hin[v] = Op::apply(M[v], Op::state_in(load_init<IO>(p, b, d_first + v, Op::default_init())));
            done = true;
            continue;
        }
        bool s_ok = true, ab_ok = true;
#pragma unroll
        for (int v = 0; v < CV; ++v) {
            s_ok = s_ok && word_valid(win.ws[i][v], p.epoch);
            ab_ok = ab_ok && word_valid(win.wa[i][v], p.epoch) && word_valid(win.wb[i][v], p.epoch);
        }
        if (s_ok) {
#pragma unroll
            for (int v = 0; v < CV; ++v) hin[v] = Op::apply(M[v], word_value(win.ws[i][v]));
            done = true;
        } else if (ab_ok) {
#pragma unroll
            for (int v = 0; v < CV; ++v)
                M[v] = Op::combine(make_float2(word_value(win.wa[i][v]), word_value(win.wb[i][v])), M[v]);
            consumed = i + 1;
        } else {
            stop = true;
        }
    }
    return done;
}

// Continue a look-back at chunk q with the running composite M (the chunks
// after q already folded in); the window of chunks q, q-1, ... is loaded.
template <class Op, typename IO, int CV, int TC, int KW>
__device__ void look_back_continue(const ScanParams &p, int64_t q, int64_t chain, int64_t b,
                                   int64_t d_first, int ch, LookWindow<CV, TC, KW> &win,
                                   float2 (&M)[CV], float (&hin)[CV]) {
    uint32_t polls = 0, ns = 32;
    while (true) {
        int consumed;
        if (resolve_window<Op, IO, CV, TC, KW>(p, q, win, b, d_first, M, hin, consumed)) return;
        if (consumed > 0) {
            q -= consumed;
            ns = 32;
        } else {
            if (++polls > p.spin_limit) {
                atomicOr(p.status, kTimeoutBit);
#pragma unroll
                for (int v = 0; v < CV; ++v) hin[v] = __int_as_float(0x7fffffff);
                return;
            }
            __nanosleep(ns);
            ns = ns < 256 ? ns * 2 : 256;
        }
        load_window<CV, TC, KW>(p, q, chain, ch, win);
    }
}

// Finish a look-back whose first window (chunks c-1 ...) is already loaded.
template <class Op, typename IO, int CV, int TC, int KW>
__device__ void look_back_from(const ScanParams &p, int64_t c, int64_t chain, int64_t b, int64_t d_first,
                               int ch, LookWindow<CV, TC, KW> &win, float (&hin)[CV]) {
    float2 M[CV];
#pragma unroll
    for (int v = 0; v < CV; ++v) M[v] = Op::identity();
    look_back_continue<Op, IO, CV, TC, KW>(p, c - 1, chain, b, d_first, ch, win, M, hin);
}

template <class Op, typename IO, int CV, int TC>
__device__ __forceinline__ void look_back(const ScanParams &p, int64_t c, int64_t chain, int64_t b,
                                          int64_t d_first, int ch, float (&hin)[CV]) {
    constexpr int KW = window_short<CV>();
    LookWindow<CV, TC, KW> win;
    load_window<CV, TC, KW>(p, c - 1, chain, ch, win);
    look_back_from<Op, IO, CV, TC, KW>(p, c, chain, b, d_first, ch, win, hin);
}

// The carry of one tile, as done by the carry warp: fold the W warp totals in
// s_tot (replaced in place by each warp's incoming state), publish the chunk
// summary, look back, publish the chunk's final state.  `between` runs after
// the per-warp states are in shared memory and before the final state is
// published (it releases the data warps).
template <class Op, typename IO, int CV, int TC, int W, class Between>
__device__ __forceinline__ void carry_tile(const ScanParams &p, int64_t tile, float2 (*s_tot)[TC],
                                           int lane, Between between) {
    const TileCoord tc = tile_coord(p, uint32_t(tile));
    const int64_t chain = tc.chain;
    const int64_t c = tc.c;
    const int64_t b = tc.b;
    const int ch = lane * CV;
    const int64_t dl = int64_t(tc.dt) * TC + ch;
    float2 total[CV];
#pragma unroll
    for (int v = 0; v < CV; ++v) total[v] = Op::identity();
    for (int w = 0; w < W; ++w) {
#pragma unroll
        for (int v = 0; v < CV; ++v) {
            const float2 t = s_tot[w][ch + v];
            s_tot[w][ch + v] = total[v];          // exclusive prefix over warps
            total[v] = Op::combine(total[v], t);
        }
    }
    const bool publish = (p.n_chunks > 1) && (c < p.n_chunks - 1) && (tile != p.drop_tile);
    float hin[CV];
    if (c == 0) {
#pragma unroll
        for (int v = 0; v < CV; ++v) hin[v] = Op::state_in(load_init<IO>(p, b, dl + v, Op::default_init()));
    } else {
        if (publish) publish_summary<CV, TC>(p, tile, ch, total);
        look_back<Op, IO, CV, TC>(p, c, chain, b, dl, ch, hin);
    }
    // state entering each warp's rows, written over the prefix pair's .x
    for (int w = 0; w < W; ++w) {
#pragma unroll
        for (int v = 0; v < CV; ++v) s_tot[w][ch + v].x = Op::apply(s_tot[w][ch + v], hin[v]);
    }
    between();
    if (publish) {
        float fin[CV];
#pragma unroll
        for (int v = 0; v < CV; ++v) fin[v] = Op::apply(total[v], hin[v]);
        publish_state<CV, TC>(p, tile, ch, fin);
    }
}

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void named_barrier_arrive(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Fold the W warp summaries of CV channels (starting at ch) into the tile
// total, replacing each summary by the exclusive prefix of the warps before it.
template <class Op, int CV, int TC, int W>
__device__ __forceinline__ void fold_warps(float2 (*s_tot)[TC], int ch, float2 (&total)[CV]) {
#pragma unroll
    for (int v = 0; v < CV; ++v) total[v] = Op::identity();
#pragma unroll
    for (int w = 0; w < W; ++w) {
#pragma unroll
        for (int v = 0; v < CV; ++v) {
            const float2 t = s_tot[w][ch + v];
            s_tot[w][ch + v] = total[v];
            total[v] = Op::combine(total[v], t);
        }
    }
}

// The tiles a block works on.  With a ticket counter (the call zeroes it on
// the stream before the launch) the block takes tickets in increasing order
// until they run out.  body(tile, take_next) runs on every thread; it calls
// take_next() once the tile's incoming state is resolved (after its own
// look-back), and thread 0 then takes the next ticket, so the atomic's
// latency hides behind the rest of the tile (the replay and stores).  A block
// never holds a ticket it has not started while it waits: every tile a
// look-back waits for is held by a running block that is working on it (or
// has finished it), and tiles wait only for smaller tickets, so waits never
// form a cycle, and a wait that gives up delays no unrelated tile.  Without
// a counter: the tile of the block's index.  Every thread of the block must
// call this; there is a block barrier between tiles.
template <class Body>
__device__ __forceinline__ void for_each_ticket(uint32_t *ticket, int64_t n_tiles, Body body) {
    if (ticket == nullptr) {
        body(int64_t(blockIdx.x), [] {});
        return;
    }
    __shared__ uint32_t s_next[2];
    if (threadIdx.x == 0) s_next[0] = atomicAdd(ticket, 1u);
    __syncthreads();
    for (int it = 0;; ++it) {
        const int64_t tile = s_next[it & 1];
        if (tile >= n_tiles) break;
        uint32_t *next = &s_next[(it + 1) & 1];
        body(tile, [&] {
            if (threadIdx.x == 0) *next = atomicAdd(ticket, 1u);
        });
        __syncthreads();                 // shared state reused by the next tile; the next ticket visible
    }
}

// -------------------------------------------------------- tile kernel
//
// One block per tile (TR rows x TC channels), W data warps + 1 carry warp.
// Template parameters: Op, IO (storage type), V (channels per thread: one
// 16-byte vector, or 1 for the scalar variant), CG (lanes across channels),
// R (rows per thread), W (data warps).  J = 32 / CG row groups per warp,
// TR = W * J * R, TC = CG * V.  Tiles are numbered chain-fastest:
// tile = chunk * n_chains + chain, chain = b * n_dt + dt.  When the sequence
// spans several chunks the blocks are persistent and take their tiles from a
// ticket counter in the workspace (for_each_ticket), so tiles are handed out
// in the order blocks reach them, whatever order the hardware dispatches
// blocks in.  Every look-back then waits only for tiles that running blocks
// hold, and a block publishes its summary before it waits, so waits never
// form a cycle.  Used for the scalar (unaligned) variant, for shapes with few
// tiles, and as a cross-check of the pipelined kernel.
template <class Op, typename IO, int V, int CG, int R, int W, int MINB>
__global__ void __launch_bounds__((W + 1) * 32, MINB) scan_tile_kernel(const ScanParams p) {
    constexpr int J = 32 / CG;
    constexpr int TR = W * J * R;
    constexpr int TC = CG * V;
    constexpr int CV = TC / 32;          // channels per carry-warp lane
    constexpr uint32_t NT = (W + 1) * 32;
    static_assert(CG * J == 32, "CG must divide 32");
    static_assert(TC % 32 == 0, "a tile spans a multiple of 32 channels");

    __shared__ float2 s_tot[W][TC];   // per-warp totals -> per-warp incoming states (.x)

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    for_each_ticket(p.ticket, p.n_tiles, [&](const int64_t tile, auto take_next) {

    if (warp < W) {
        const TileCoord tc = tile_coord(p, uint32_t(tile));
        const int64_t c = tc.c;
        const int64_t b = tc.b;
        const int64_t dt = tc.dt;
        const int g = lane % CG;
        const int j = lane / CG;
        const int64_t d0 = dt * TC + int64_t(g) * V;
        const bool dvalid = d0 < p.D;            // V > 1 requires D % V == 0
        const int64_t row0 = c * TR + int64_t(warp * J + j) * R;
        const IO *in0 = static_cast<const IO *>(p.in0);
        const IO *in1 = static_cast<const IO *>(p.in1);
        IO *out = static_cast<IO *>(p.out);
        const int64_t base = (b * p.T) * p.D + d0;

        float x0[R][V], x1[R][V];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t t = row0 + r;
            if (dvalid && t < p.T) {
                Access<IO, V>::load(in0 + base + t * p.D, x0[r]);
                Access<IO, V>::load(in1 + base + t * p.D, x1[r]);
            } else {
#pragma unroll
                for (int v = 0; v < V; ++v) { x0[r][v] = Op::pad0(); x1[r][v] = Op::pad1(); }
            }
        }
        float2 incl[V];
#pragma unroll
        for (int v = 0; v < V; ++v) incl[v] = Op::identity();
        [[maybe_unused]] float lam2[V];
        if constexpr (Op::kDecay) {
#pragma unroll
            for (int v = 0; v < V; ++v) lam2[v] = decay_lam2(p, d0 + v);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            [[maybe_unused]] float u = 0.f;        // rows past T: gamma = 1 keeps the padding pair the identity
            if constexpr (Op::kDecay) {
                if (row0 + r < p.T) u = decay_u(p, b, row0 + r);
            }
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float e0, e1;
                Op::element(x0[r][v], x1[r][v], e0, e1);
                if constexpr (Op::kDecay) e0 *= decay_gamma(lam2[v], u);
                x0[r][v] = e0;
                x1[r][v] = e1;
                incl[v] = Op::combine(incl[v], make_float2(e0, e1));
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
        float2 excl[V];   // exclusive within the warp
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float2 o;
            o.x = __shfl_up_sync(0xffffffffu, incl[v].x, CG);
            o.y = __shfl_up_sync(0xffffffffu, incl[v].y, CG);
            excl[v] = (J > 1 && j > 0) ? o : Op::identity();
        }
        named_barrier_sync(1, NT);   // totals are in shared memory
        named_barrier_sync(2, NT);   // the carry warp has written the warp states
        take_next();                 // the tile's look-back is over: take the next ticket

        float st[V];
#pragma unroll
        for (int v = 0; v < V; ++v) st[v] = Op::apply(excl[v], s_tot[warp][g * V + v].x);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float y[V];
#pragma unroll
            for (int v = 0; v < V; ++v) {
                st[v] = Op::step(x0[r][v], x1[r][v], st[v]);
                y[v] = Op::state_out(st[v]);
            }
            const int64_t t = row0 + r;
            if (dvalid && t < p.T) Access<IO, V>::store(out + base + t * p.D, y);
        }
    } else {
        named_barrier_sync(1, NT);
        carry_tile<Op, IO, CV, TC, W>(p, tile, s_tot, lane, [&] { named_barrier_sync(2, NT); });
    }
    });
}

// --------------------------------------------------- pipelined kernel
//
// Persistent blocks (co-resident, cooperative launch), each owning tiles
// blockIdx.x, blockIdx.x + gridDim.x, ... in order: 7 data warps and one
// carry warp with two blocks per SM, or 15 and one with one block per SM.  A tile is TR x TC with TC = CG * V channels (V = 4) and
// TR = W * J * R rows (J = 32 / CG row groups per warp): lane (g, j) =
// (lane % CG, lane / CG) of warp w owns channels [g V, g V + V) of rows
// [(w J + j) R, (w J + j) R + R).  Narrow tiles (128-byte rows) keep the chunk
// hand-off cheap: about gridDim.x / n_chains chunks of one channel tile are in
// flight at once, and a look-back folds that many summaries of TC channels.
//
// Loads: the tensor memory accelerator copies whole tiles (box TC x TR x 1 of
// the (D, T, B) tensor) of both operands into an S-slot shared-memory ring,
// an mbarrier per slot counting the bytes in.  The carry warp issues the
// first S tiles; afterwards the last data warp to finish reading a slot (a
// shared counter per slot) issues the next tile into it at once.  Rows past T
// and channels past D arrive as zeros and are replaced by the operator's
// identity inputs in registers.  No multicast.
//
// Compute, with a one-tile lag: phase A of tile n (activations, the thread's
// fold over its R rows, the scan across the warp's J row groups, the warp's
// summary to shared memory; pairs and the thread's exclusive prefix stay in
// registers), then phase B of tile n-1 (replay from the thread's incoming
// state, streaming stores).  With R = 8 rows per thread two tiles' pairs no
// longer fit in registers, and phase B of tile n follows its own phase A.
//
// Carry warp: it resolves tile n's incoming state (a look-back over earlier
// chunks only) while the data warps are still in phase A of tile n, so once
// tile n's summaries are in it only writes the state and releases them; the
// loads of tile n+1's look-back window are issued as soon as tile n is
// released.  Named barriers and summaries are double-buffered by tile parity:
//   barrier 1 + (n & 1): data warps arrive (summaries of tile n written),
//                        carry warp waits;
//   barrier 3 + (n & 1): carry warp arrives (incoming states of tile n
//                        written), data warps wait (phase B of n).
// Data warps reach phase A of n only after phase B of n-2, which the carry
// warp released before it waited for tile n-1: no cycle.  Every look-back
// wait is for a tile with a smaller index and blocks are co-resident, so the
// smallest unfinished tile can always progress.
template <typename IO, int V, int CG, int R, int S, int W, bool DEC = false>
struct PipeShape {
    static constexpr int J = 32 / CG;
    static constexpr int TC = CG * V;
    static constexpr int TR = W * J * R;
    static constexpr size_t op_bytes = size_t(TR) * TC * sizeof(IO);     // one operand of a tile
    // time decay through the copy engine: the tile's TC rates, then its TR
    // row gaps (fp32), follow the two operands in the slot.  Every copy's
    // shared-memory destination must sit on a 128-byte boundary, a copy box
    // spans at most 256 elements a dimension and 16-byte multiples of them,
    // and a gap box starts at a row index whose byte offset is a multiple
    // of 16 (tiles start at multiples of TR).
    static constexpr bool dec_boxable = TR % 4 == 0 && TR <= 256 && TC <= 256 && (TC * 4) % 128 == 0;
    static_assert(op_bytes % 128 == 0, "operand copies land on 128-byte boundaries");
    static constexpr size_t dec_bytes = DEC ? size_t(TR + TC) * sizeof(float) : 0;
    static constexpr size_t tx_bytes = 2 * op_bytes + dec_bytes;         // bytes a tile's copies bring
    static constexpr size_t slot_bytes = (tx_bytes + 127) / 128 * 128;
    static constexpr size_t bar_offset = S * slot_bytes;
    static constexpr size_t cnt_offset = bar_offset + S * 8;          // per-slot reader counts
    static constexpr size_t tot_offset = (cnt_offset + S * 4 + 15) / 16 * 16;        // [2][W][TC] float2
    static constexpr size_t total_offset = tot_offset + size_t(2) * W * TC * sizeof(float2);  // [2][TC] float2
    static constexpr size_t hin_offset = total_offset + size_t(2) * TC * sizeof(float2);     // [2][TC] float
    static constexpr size_t smem_bytes = hin_offset + size_t(2) * TC * sizeof(float);
};

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// bounded wait for a phase of an mbarrier; false if it did not complete
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}
// 3-D tiled tensor load into this block's shared memory, completion counted
// on an mbarrier (plain load: no cluster multicast)
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y, int z,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void tma_load_1d(uint32_t dst, const CUtensorMap *map, int x, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.1d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2}], [%3];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(bar) : "memory");
}

// bound on mbarrier polls (each try_wait may suspend the thread for up to a
// microsecond or so); after one wait has run out, later waits of the thread
// make a single poll, so a broken copy cannot stretch the kernel to n_local
// full bounds
constexpr uint32_t kMbarLimit = 1u << 16;

// DT (time decay only): the gaps and rates come with the tile through the
// copy engine (map_gap: the (B, T) gaps, map_lam: the (D,) rates), so they
// hold no registers across the wait and the one-tile lag fits; otherwise
// they are plain loads and map_gap, map_lam are unused.
template <class Op, typename IO, int V, int CG, int R, int S, int W, int MINB, bool DT = false>
__global__ void __launch_bounds__((W + 1) * 32, MINB)
scan_pipelined_kernel(const ScanParams p, const __grid_constant__ CUtensorMap map0,
                      const __grid_constant__ CUtensorMap map1, const __grid_constant__ CUtensorMap map_gap,
                      const __grid_constant__ CUtensorMap map_lam) {
    static_assert(!DT || Op::kDecay, "decay operands through the copy engine need a decay operator");
    using Shape = PipeShape<IO, V, CG, R, S, W, DT>;
    static_assert(!DT || Shape::dec_boxable, "decay operands fit copy boxes");
    using Vec = typename VecOf<IO, V>::type;
    constexpr int J = Shape::J;
    constexpr int TC = Shape::TC;
    constexpr int TR = Shape::TR;
    constexpr int CV = TC / 32;
    constexpr uint32_t NT = (W + 1) * 32;
    // Who folds the W warp summaries into the tile total and publishes the
    // chunk summary: with fp32 I/O the carry warp's per-tile work is the
    // limit, so the last data warp of the tile does it; with bf16 I/O (half
    // the bytes per element) the data warps' instruction issue is the limit,
    // so the carry warp does it.
    constexpr bool kFoldInData = sizeof(IO) == 4;
    // Phase B of a tile runs one tile late (LAG) so the data warps never wait
    // for the carry warp, at the price of holding two tiles' pairs in
    // registers; with 8 rows per thread that no longer fits, so those tiles
    // replay right after their own phase A and the per-tile work (warp scan,
    // barriers, tile coordinates) is spread over twice the elements.  The
    // time-decay gate's per-channel rates and per-row gaps do not fit beside
    // two tiles' pairs either (register spills measured slower than waiting).
    constexpr bool LAG = R < 8 && (!Op::kDecay || DT);
    constexpr int NB = LAG ? 2 : 1;
    static_assert(sizeof(Vec) == V * sizeof(IO), "vector type matches the vector width");
    static_assert(CG * J == 32 && TC % 32 == 0, "lane layout");
    static_assert(TC * sizeof(IO) % 16 == 0 && TC <= 256 && TR <= 256, "TMA box");

    extern __shared__ __align__(128) unsigned char smem[];
    float2 (*s_tot)[W][TC] = reinterpret_cast<float2 (*)[W][TC]>(smem + Shape::tot_offset);
    float2 (*s_total)[TC] = reinterpret_cast<float2 (*)[TC]>(smem + Shape::total_offset);
    float (*s_hin)[TC] = reinterpret_cast<float (*)[TC]>(smem + Shape::hin_offset);
    unsigned int *s_cnt = reinterpret_cast<unsigned int *>(smem + Shape::cnt_offset);
    const uint32_t ring = smem_addr(smem);
    const uint32_t bars = ring + uint32_t(Shape::bar_offset);

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t G = gridDim.x;
    const int64_t first = blockIdx.x;
    const int n_local = int((p.n_tiles - first + G - 1) / G);

    // TMA copy of tile n into ring slot n % S (one thread)
    auto issue_tile = [&](int n) {
        const TileCoord tc = tile_coord(p, uint32_t(first + int64_t(n) * G));
        const uint32_t slot = ring + uint32_t((n % S) * Shape::slot_bytes);
        const uint32_t bar = bars + 8u * uint32_t(n % S);
        const int x = int(tc.dt) * TC, y = int(tc.c) * TR, z = int(tc.b);
        mbar_expect_tx(bar, uint32_t(Shape::tx_bytes));
        tma_load_3d(slot, &map0, x, y, z, bar);
        tma_load_3d(slot + uint32_t(Shape::op_bytes), &map1, x, y, z, bar);
        if constexpr (DT) {
            tma_load_1d(slot + uint32_t(2 * Shape::op_bytes), &map_lam, x, bar);
            tma_load_2d(slot + uint32_t(2 * Shape::op_bytes) + uint32_t(TC) * 4u, &map_gap, y, z, bar);
        }
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(bars + 8u * s, 1);
            s_cnt[s] = 0;
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
        IO *out = static_cast<IO *>(p.out);
        constexpr int V2 = V / 2;

        // pairs of the tiles in flight (two with the lag, by tile parity), two
        // channels per float2
        float2 PA[NB][R][V2], PB[NB][R][V2];
        float2 E[NB][V];     // the thread's exclusive prefix within its warp, per channel
        // per tile buffer, what phase B needs: the thread's first output
        // element and how many of its R rows lie inside the tensor (0 for
        // channels past D)
        IO *dstb[NB];
        int nval[NB];
        uint32_t wait_limit = kMbarLimit;

        auto phaseA = [&](int n, auto bufc) {
            constexpr int BUF = decltype(bufc)::value;
            constexpr int SB = LAG ? BUF : 0;
            const TileCoord tc = tile_coord(p, uint32_t(first + int64_t(n) * G));
            const int64_t d0 = int64_t(tc.dt) * TC + g * V;
            const bool dvalid = d0 < p.D;
            const int row0 = int(tc.c) * TR + (warp * J + j) * R;
            const int64_t left = p.T - row0;
            nval[SB] = dvalid ? int(left < R ? (left > 0 ? left : 0) : R) : 0;
            const bool full = nval[SB] == R;
            dstb[SB] = out + (int64_t(tc.b) * p.T + row0) * p.D + d0;
            // time decay: the tile's rates and the thread's row gaps are plain
            // global loads, issued before the wait for the tile so that their
            // latency overlaps it
            [[maybe_unused]] float lam2[V], ur[R];
            if constexpr (Op::kDecay && !DT) {
#pragma unroll
                for (int v = 0; v < V; ++v) lam2[v] = decay_lam2(p, d0 + v);
#pragma unroll
                for (int r = 0; r < R; ++r) ur[r] = row0 + r < p.T ? decay_u(p, tc.b, row0 + r) : 0.f;
            }
            if (!mbar_wait(bars + 8u * uint32_t(n % S), uint32_t((n / S) & 1), wait_limit)) {
                wait_limit = 1;
                if (lane == 0 && p.status) atomicOr(p.status, kTimeoutBit);   // null: one chunk, no workspace
            }
            const IO *t0 = reinterpret_cast<const IO *>(smem + (n % S) * Shape::slot_bytes) +
                           ((warp * J + j) * R) * TC + g * V;
            const IO *t1 = t0 + TR * TC;
            // DT: the tile's rates (channels past D read 0) and gaps (rows
            // past T read 0: gamma = 1) in the slot
            [[maybe_unused]] const float *s_lam =
                reinterpret_cast<const float *>(smem + (n % S) * Shape::slot_bytes + 2 * Shape::op_bytes);
            [[maybe_unused]] const float *s_gap = s_lam + TC;
            // DT: the thread's rates (as lam2 pairs) and its R row gaps, read
            // once per tile
            [[maybe_unused]] float2 l2p[V2];
            if constexpr (DT) {
#pragma unroll
                for (int i = 0; i < V2; ++i)
                    l2p[i] = __fmul2_rn(*reinterpret_cast<const float2 *>(s_lam + g * V + 2 * i),
                                        make_float2(kNegLog2e, kNegLog2e));
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    ur[r] = s_gap[(warp * J + j) * R + r];
                    if (p.decay_log1p) ur[r] = log1pf(ur[r]);
                }
            }
            float2 IA[V2], IB[V2];
#pragma unroll
            for (int i = 0; i < V2; ++i) {
                IA[i] = make_float2(Op::identity().x, Op::identity().x);
                IB[i] = make_float2(Op::identity().y, Op::identity().y);
            }
            auto rows = [&](auto fullc) {
                constexpr bool FULL = decltype(fullc)::value;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    float x0[V], x1[V];
                    unpack(*reinterpret_cast<const Vec *>(t0 + r * TC), x0);
                    unpack(*reinterpret_cast<const Vec *>(t1 + r * TC), x1);
                    [[maybe_unused]] float u = 0.f;
                    if constexpr (Op::kDecay) u = ur[r];
                    if (!FULL) {
                        const bool ok = r < nval[SB];
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            x0[v] = ok ? x0[v] : Op::pad0();
                            x1[v] = ok ? x1[v] : Op::pad1();
                        }
                    }
#pragma unroll
                    for (int i = 0; i < V2; ++i) {
                        float2 a2, b2;
                        element_pair<Op, IO>(x0[2 * i], x1[2 * i], x0[2 * i + 1], x1[2 * i + 1], a2, b2);
                        if constexpr (DT) {
                            const float2 e = __fmul2_rn(l2p[i], make_float2(u, u));
                            a2 = __fmul2_rn(a2, make_float2(fast_exp2(e.x), fast_exp2(e.y)));
                        } else if constexpr (Op::kDecay) {
                            a2 = __fmul2_rn(a2, make_float2(decay_gamma(lam2[2 * i], u), decay_gamma(lam2[2 * i + 1], u)));
                        }
                        PA[SB][r][i] = a2;
                        PB[SB][r][i] = b2;
                        Op::fold2(IA[i], IB[i], a2, b2);
                    }
                }
            };
            if (full) rows(std::true_type{});
            else rows(std::false_type{});
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
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float2 o;
                o.x = __shfl_up_sync(0xffffffffu, incl[v].x, CG);
                o.y = __shfl_up_sync(0xffffffffu, incl[v].y, CG);
                E[SB][v] = (J > 1 && j > 0) ? o : Op::identity();
            }
            if (j == J - 1) {
#pragma unroll
                for (int v = 0; v < V; ++v) s_tot[BUF][warp][g * V + v] = incl[v];
            }
            // The warp is done with the slot and has written its summary.  The
            // last of the W warps (a shared counter per slot) refills the slot
            // with tile n + S and, for fp32 I/O, folds the W warp summaries
            // into per-warp exclusive prefixes and the tile total and publishes
            // the chunk summary, so the carry warp only has the look-back left.
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
                    const int64_t tile = first + int64_t(n) * G;
                    const bool publish =
                        (p.n_chunks > 1) && (int64_t(tc.c) < p.n_chunks - 1) && (tile != p.drop_tile);
                    if (publish && tc.c > 0) publish_summary<CV, TC>(p, tile, ch, total);
                }
            }
            named_barrier_arrive(1 + BUF, NT);
        };

        auto phaseB = [&](auto bufc) {
            constexpr int BUF = decltype(bufc)::value;
            constexpr int SB = LAG ? BUF : 0;
            named_barrier_sync(3 + BUF, NT);
            float2 st[V2];
#pragma unroll
            for (int i = 0; i < V2; ++i) {
                const int c0 = g * V + 2 * i;
                const float w0 = Op::apply(s_tot[BUF][warp][c0], s_hin[BUF][c0]);
                const float w1 = Op::apply(s_tot[BUF][warp][c0 + 1], s_hin[BUF][c0 + 1]);
                st[i] = make_float2(Op::apply(E[SB][2 * i], w0), Op::apply(E[SB][2 * i + 1], w1));
            }
            IO *dst = dstb[SB];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float y[V];
#pragma unroll
                for (int i = 0; i < V2; ++i) {
                    st[i] = Op::step2(PA[SB][r][i], PB[SB][r][i], st[i]);
                    y[2 * i] = Op::state_out(st[i].x);
                    y[2 * i + 1] = Op::state_out(st[i].y);
                }
                if (r < nval[SB]) Access<IO, V>::store(dst, y);
                dst += p.D;
            }
        };

        using B0 = std::integral_constant<int, 0>;
        using B1 = std::integral_constant<int, 1>;
        int n = 0;
        if constexpr (LAG) {
            for (; n + 1 < n_local; n += 2) {
                phaseA(n, B0{});
                if (n >= 1) phaseB(B1{});
                phaseA(n + 1, B1{});
                phaseB(B0{});
            }
            if (n < n_local) {
                phaseA(n, B0{});
                if (n >= 1) phaseB(B1{});
                phaseB(B0{});
            } else if (n_local >= 1) {
                phaseB(B1{});
            }
        } else {
            for (; n + 1 < n_local; n += 2) {
                phaseA(n, B0{});
                phaseB(B0{});
                phaseA(n + 1, B1{});
                phaseB(B1{});
            }
            if (n < n_local) {
                phaseA(n, B0{});
                phaseB(B0{});
            }
        }
    } else {
        // ============================================== carry warp
        // Per tile: resolve the incoming state from the look-back window
        // (issued when the previous tile was done) while the data warps are in
        // phase A; wait for the tile's warp summaries; (bf16 I/O: fold them and
        // publish the chunk summary;) write the incoming state, release the
        // data warps, publish the chunk's final state, and issue the next
        // tile's look-back loads.  A look-back only ever waits for chunks with
        // smaller tile indices, whose blocks never wait on this one.
        const int ch = lane * CV;
        constexpr int KW = window_long<CV>();
        LookWindow<CV, TC, KW> win;
        float init[CV];
        auto prefetch = [&](int n) {
            const TileCoord tc = tile_coord(p, uint32_t(first + int64_t(n) * G));
            if (tc.c == 0) {
#pragma unroll
                for (int v = 0; v < CV; ++v)
                    init[v] = Op::state_in(load_init<IO>(p, tc.b, int64_t(tc.dt) * TC + ch + v, Op::default_init()));
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
            // The incoming state depends only on earlier chunks: resolve it
            // while the data warps are still in phase A of this tile.  When
            // this warp publishes the tile's summary itself (bf16), it must not
            // wait for earlier chunks first -- the next chunk's look-back may
            // be waiting for that summary, and waiting here would chain the
            // chunks of a channel tile one after another -- so it only walks
            // the window already loaded and finishes the walk after publishing.
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

// ------------------------------------------------ sequence summaries
//
// For a time axis split across devices (each holds a contiguous slice), the
// one exchange a scan needs is each slice's summary: per channel, the
// composition of all its steps' pairs (minGRU: h_end = A h_start + B; MinMax:
// x_end = max(min(x_start, U), L)).  Pass 1 folds segments of `seg` rows per
// thread (one thread per V channels of one segment, rows walked in order) into
// partial pairs [n_seg][B][D]; pass 2 folds each channel's partials in segment
// order into [B][D] pairs.  Both read every input once; no state crosses
// blocks, so there is no hand-off and no waiting.
template <class Op, typename IO, int V>
__global__ void __launch_bounds__(256) scan_summary_kernel(const ScanParams p, int64_t seg,
                                                           int64_t n_seg, float2 *partial) {
    constexpr int U = V >= 8 ? 2 : (V >= 4 ? 4 : 8);           // rows loaded ahead per thread
    const int64_t groups = (p.D + V - 1) / V;                 // channel groups per batch row
    const int64_t n = p.B * groups * n_seg;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t gch = i % groups;                        // channel group fastest: coalesced rows
        const int64_t rest = i / groups;
        const int64_t b = rest % p.B;
        const int64_t sg = rest / p.B;
        const int64_t d0 = gch * V;
        const int64_t t0 = sg * seg;
        const int64_t t1 = t0 + seg < p.T ? t0 + seg : p.T;
        const IO *in0 = static_cast<const IO *>(p.in0);
        const IO *in1 = static_cast<const IO *>(p.in1);
        const bool whole = d0 + V <= p.D;
        float2 acc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = Op::identity();
        [[maybe_unused]] float lam2[V];
        if constexpr (Op::kDecay) {
#pragma unroll
            for (int v = 0; v < V; ++v) lam2[v] = decay_lam2(p, d0 + v);
        }
        for (int64_t t = t0; t < t1; t += U) {
            // all U rows' loads first (memory-level parallelism), then the fold
            float x0[U][V], x1[U][V];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t off = (b * p.T + t + u) * p.D + d0;
                if (t + u < t1 && whole) {
                    Access<IO, V>::load(in0 + off, x0[u]);
                    Access<IO, V>::load(in1 + off, x1[u]);
                } else {
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        const bool ok = t + u < t1 && d0 + v < p.D;
                        x0[u][v] = ok ? load_scalar<IO>(in0 + off + v) : Op::pad0();
                        x1[u][v] = ok ? load_scalar<IO>(in1 + off + v) : Op::pad1();
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                [[maybe_unused]] float gu = 0.f;
                if constexpr (Op::kDecay) gu = (t + u < t1) ? decay_u(p, b, t + u) : 0.f;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    float e0, e1;
                    Op::element(x0[u][v], x1[u][v], e0, e1);
                    if constexpr (Op::kDecay) e0 *= decay_gamma(lam2[v], gu);
                    acc[v] = Op::combine(acc[v], make_float2(e0, e1));
                }
            }
        }
#pragma unroll
        for (int v = 0; v < V; ++v) {
            if (d0 + v < p.D) partial[(sg * p.B + b) * p.D + d0 + v] = acc[v];
        }
    }
}

// out[g][i] = the pairs partial[g G .. g G + G - 1][i] folded in order (the
// last group may be shorter); one thread per (group, channel), channels
// fastest so that every load of a segment's pairs is coalesced.
template <class Op>
__global__ void __launch_bounds__(256) fold_partials_kernel(const float2 *partial, int64_t n_seg,
                                                            int64_t G, int64_t BD, float2 *out) {
    const int64_t n_groups = (n_seg + G - 1) / G;
    const int64_t n = (n_groups > 0 ? n_groups : 1) * BD;
    for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < n;
         idx += int64_t(gridDim.x) * blockDim.x) {
        const int64_t grp = idx / BD, i = idx - grp * BD;
        const int64_t s0 = grp * G;
        const int64_t s1 = s0 + G < n_seg ? s0 + G : n_seg;
        float2 acc = Op::identity();
        int64_t sg = s0;
        for (; sg + 8 <= s1; sg += 8) {             // eight loads in flight, then fold in order
            float2 x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] = partial[(sg + u) * BD + i];
#pragma unroll
            for (int u = 0; u < 8; ++u) acc = Op::combine(acc, x[u]);
        }
        for (; sg < s1; ++sg) acc = Op::combine(acc, partial[sg * BD + i]);
        out[grp * BD + i] = acc;
    }
}

// Incoming state of slice `rank`: the summaries of slices 0 .. rank-1 (stored
// [n_slices][B][D] pairs) applied in order to the initial state (null:
// the operator's default), written in the I/O type.
template <class Op, typename IO>
__global__ void __launch_bounds__(256) combine_summaries_kernel(const float2 *pairs, int64_t rank,
                                                                const IO *init, int64_t init_bs,
                                                                IO *out, int64_t out_bs, int64_t B,
                                                                int64_t D) {
    const int64_t BD = B * D;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < BD;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t b = i / D, d = i - b * D;
        float x = init ? load_scalar<IO>(init + b * init_bs + d) : Op::default_init();
        for (int64_t r = 0; r < rank; ++r) x = Op::apply(pairs[r * BD + i], x);
        const float y[1] = {x};
        Access<IO, 1>::store(out + b * out_bs + d, y);
    }
}

// ------------------------------------------------------------ step kernel
//
// One token for (B, D) rows: the same per-element arithmetic as the scan's
// phase 1 and phase 3, so a parallel prefix followed by steps reproduces the
// scan to fp32 rounding.
template <typename IO>
__global__ void __launch_bounds__(256) mingru_step_kernel(
    const IO *__restrict__ k, int64_t k_bs, const IO *__restrict__ hx, int64_t hx_bs,
    const IO *h_prev, int64_t hp_bs, IO *h_out, int64_t ho_bs, int64_t B, int64_t D) {
    const int64_t n = B * D;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t b = i / D;
        const int64_t d = i - b * D;
        const float kv = load_scalar<IO>(k + b * k_bs + d);
        const float hv = load_scalar<IO>(hx + b * hx_bs + d);
        float a, bb;
        MinGRUOp::element(kv, hv, a, bb);
        const float prev = h_prev ? load_scalar<IO>(h_prev + b * hp_bs + d) : 0.f;
        float y[1] = {MinGRUOp::step(a, bb, prev)};
        if constexpr (sizeof(IO) == 4) {
            h_out[b * ho_bs + d] = y[0];
        } else {
            h_out[b * ho_bs + d] = __float2bfloat16_rn(y[0]);
        }
    }
}

}  // namespace sgr
