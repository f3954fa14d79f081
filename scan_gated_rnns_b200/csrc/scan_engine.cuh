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
// (no cancellation: all terms are positive) and with 3 MUFU ops per element
// instead of about 7.
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
#include <stdint.h>

namespace sgr {

// ------------------------------------------------------------- operators

struct MinGRUOp {
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
    // Both sigmoids come from e = exp(-|x|) in (0, 1]: sigmoid(|x|) = 1/(1+e),
    // sigmoid(-|x|) = e/(1+e); the two reciprocals share one division.
    static __device__ __forceinline__ void element(float k, float hx, float &a, float &b) {
        const float ek = __expf(-fabsf(k));
        const float eh = __expf(-fabsf(hx));
        const float dk = 1.f + ek;
        const float dh = 1.f + eh;
        const float inv = __frcp_rn(dk * dh);
        const float rk = dh * inv;   // 1 / (1 + ek)
        const float rh = dk * inv;   // 1 / (1 + eh)
        const float ekr = ek * rk;
        const bool kpos = k >= 0.f;
        const float z = kpos ? rk : ekr;
        a = kpos ? ekr : rk;
        const float g = (hx >= 0.f) ? hx + 0.5f : eh * rh;
        b = z * g;
    }
    // one step of phase 3
    static __device__ __forceinline__ float step(float a, float b, float x) { return fmaf(a, x, b); }
    // initial state when none is given
    static __device__ __forceinline__ float default_init() { return 0.f; }
};

struct MinMaxOp {
    // pair (U, L): state -> max(min(state, U), L)
    static __device__ __forceinline__ float2 identity() { return make_float2(INFINITY, -INFINITY); }
    static __device__ __forceinline__ float2 combine(float2 p, float2 q) {
        return make_float2(fminf(p.x, q.x), fmaxf(fminf(p.y, q.x), q.y));
    }
    static __device__ __forceinline__ float apply(float2 p, float x) { return fmaxf(fminf(x, p.x), p.y); }
    static __device__ __forceinline__ float pad0() { return INFINITY; }
    static __device__ __forceinline__ float pad1() { return -INFINITY; }
    static __device__ __forceinline__ void element(float r, float s, float &u, float &l) { u = r; l = s; }
    static __device__ __forceinline__ float step(float u, float l, float x) { return fmaxf(fminf(x, u), l); }
    static __device__ __forceinline__ float default_init() { return 0.f; }
};

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

// ------------------------------------------------------- look-back plumbing

__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(uint64_t *p, uint64_t v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Chunk status word: (epoch << 2) | state.  The epoch is new for every launch,
// so words left by earlier launches read as "not ready".
enum : uint32_t { ST_NONE = 0, ST_AGG = 1, ST_PREFIX = 2 };

// bounded waiting: 2^18 polls with back-off capped at 1 us => a fraction of a
// second, far above the microseconds a chunk waits for a running predecessor
constexpr uint32_t kSpinLimit = 1u << 18;
constexpr uint32_t kTimeoutBit = 1u;

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
    uint64_t *flags;      // [n_chunks * n_chains] status words (workspace)
    float2 *agg;          // [n_chunks * n_chains * TC] chunk summaries
    float *pref;          // [n_chunks * n_chains * TC] state at the end of each chunk
    uint32_t *status;     // device status word
    uint64_t epoch;
    uint32_t spin_limit;  // polls before a chunk gives up waiting
    int64_t drop_tile;    // testing: this tile does not publish (-1: none)
};

// ----------------------------------------------------------------- kernel
//
// Template parameters: Op (operator), IO (storage type), V (channels per thread,
// one 16-byte vector or 1), CG (lanes across channels), R (rows per thread),
// W (data warps).  J = 32 / CG row groups per warp.  Tile = TR x TC with
// TR = W * J * R rows and TC = CG * V channels.
//
// The block has W data warps and one carry warp.  Data warps hold the tile in
// registers; the carry warp holds none and does the cross-chunk work (publish
// the chunk summary, look back, publish the chunk's final state).  The two
// roles sit in disjoint branches that meet only at named barriers, so their
// register live ranges never add up.
//
// Tiles are numbered chain-fastest: blockIdx.x = chunk * n_chains + chain,
// chain = b * n_dt + dt.  Blocks are dispatched in increasing index order, so
// every chunk a block waits for belongs to a block that started earlier; a
// block publishes its summary before it waits, so waits never form a cycle.

__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <class Op, typename IO, int V, int CG, int R, int W, int MINB>
__global__ void __launch_bounds__((W + 1) * 32, MINB) scan_kernel(const ScanParams p) {
    constexpr int J = 32 / CG;
    constexpr int TR = W * J * R;
    constexpr int TC = CG * V;
    constexpr int CV = TC / 32;          // channels per carry-warp lane
    constexpr uint32_t NT = (W + 1) * 32;
    static_assert(CG * J == 32, "CG must divide 32");
    static_assert(TC % 32 == 0, "a tile spans a multiple of 32 channels");

    __shared__ float2 s_tot[W][TC];   // per-warp totals, then per-warp exclusive prefixes
    __shared__ float s_win[W][TC];    // state entering each warp's rows

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;

    const int64_t tile = blockIdx.x;
    const int64_t chain = tile % p.n_chains;
    const int64_t c = tile / p.n_chains;
    const int64_t b = chain / p.n_dt;
    const int64_t dt = chain - b * p.n_dt;

    if (warp < W) {
        // ================================================= data warps
        const int g = lane % CG;
        const int j = lane / CG;
        const int64_t d0 = dt * TC + int64_t(g) * V;
        const bool dvalid = d0 < p.D;            // V > 1 requires D % V == 0
        const int64_t row0 = c * TR + int64_t(warp * J + j) * R;
        const IO *in0 = static_cast<const IO *>(p.in0);
        const IO *in1 = static_cast<const IO *>(p.in1);
        IO *out = static_cast<IO *>(p.out);
        const int64_t base = (b * p.T) * p.D + d0;

        // ---- load R rows x V channels of both operands (all in flight at once)
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

        // ---- phase 1: activations and the thread's own fold
        float2 incl[V];
#pragma unroll
        for (int v = 0; v < V; ++v) incl[v] = Op::identity();
#pragma unroll
        for (int r = 0; r < R; ++r) {
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float e0, e1;
                Op::element(x0[r][v], x1[r][v], e0, e1);
                x0[r][v] = e0;
                x1[r][v] = e1;
                incl[v] = Op::combine(incl[v], make_float2(e0, e1));
            }
        }

        // ---- phase 2a: inclusive scan across the J row groups of the warp
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
        named_barrier(1, NT);   // totals are in shared memory
        named_barrier(2, NT);   // the carry warp has filled s_win

        // ---- phase 3: replay the thread's steps from its incoming state, store
        float st[V];
#pragma unroll
        for (int v = 0; v < V; ++v) st[v] = Op::apply(excl[v], s_win[warp][g * V + v]);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float y[V];
#pragma unroll
            for (int v = 0; v < V; ++v) {
                st[v] = Op::step(x0[r][v], x1[r][v], st[v]);
                y[v] = st[v];
            }
            const int64_t t = row0 + r;
            if (dvalid && t < p.T) Access<IO, V>::store(out + base + t * p.D, y);
        }
    } else {
        // ================================================= carry warp
        // lane owns tile channels [lane * CV, lane * CV + CV)
        const int ch = lane * CV;
        const int64_t dl = dt * TC + ch;   // first global channel
        float init[CV];
#pragma unroll
        for (int v = 0; v < CV; ++v) {
            init[v] = Op::default_init();
            if (p.init != nullptr && dl + v < p.D)
                init[v] = load_scalar<IO>(static_cast<const IO *>(p.init) + b * p.init_bs + dl + v);
        }
        named_barrier(1, NT);

        // exclusive prefix over the warps (in place) and the tile total
        float2 total[CV];
#pragma unroll
        for (int v = 0; v < CV; ++v) total[v] = Op::identity();
        for (int w = 0; w < W; ++w) {
#pragma unroll
            for (int v = 0; v < CV; ++v) {
                const float2 t = s_tot[w][ch + v];
                s_tot[w][ch + v] = total[v];
                total[v] = Op::combine(total[v], t);
            }
        }

        float hin[CV];
#pragma unroll
        for (int v = 0; v < CV; ++v) hin[v] = init[v];
        const int64_t slot = tile;
        const bool publish = (p.n_chunks > 1) && (c < p.n_chunks - 1) && (tile != p.drop_tile);
        const uint64_t tag = p.epoch << 2;
        if (c > 0) {
            // publish this chunk's summary so later chunks need not wait for its carry
            if (publish) {
#pragma unroll
                for (int v = 0; v < CV; ++v) __stcg(&p.agg[slot * TC + ch + v], total[v]);
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_u64(&p.flags[slot], tag | ST_AGG);
            }
            // decoupled look-back: lane i watches chunk pos - i
            float2 M[CV];
#pragma unroll
            for (int v = 0; v < CV; ++v) M[v] = Op::identity();
            int64_t pos = c - 1;
            uint32_t polls = 0;
            bool timed_out = false;
            while (true) {
                const int64_t q = pos - lane;
                int first = 32;
                uint32_t ns = 32;
                while (true) {
                    uint32_t stt = ST_PREFIX;   // before chunk 0: the initial state
                    if (q >= 0) {
                        const uint64_t f = ld_acquire_u64(&p.flags[q * p.n_chains + chain]);
                        stt = ((f >> 2) == p.epoch) ? uint32_t(f & 3u) : ST_NONE;
                    }
                    const uint32_t pm = __ballot_sync(0xffffffffu, stt == ST_PREFIX);
                    const uint32_t rm = __ballot_sync(0xffffffffu, stt != ST_NONE);
                    first = pm ? (__ffs(pm) - 1) : 32;
                    const uint32_t need = (first >= 31) ? 0xffffffffu : ((2u << first) - 1u);
                    if ((rm & need) == need) break;
                    if (++polls > p.spin_limit) { timed_out = true; break; }
                    __nanosleep(ns);
                    ns = ns < 1024 ? ns * 2 : 1024;
                }
                __syncwarp();
                if (timed_out) break;
                for (int i = 0; i < first; ++i) {
                    const int64_t qq = pos - i;
#pragma unroll
                    for (int v = 0; v < CV; ++v) {
                        const float2 a = __ldcg(&p.agg[(qq * p.n_chains + chain) * TC + ch + v]);
                        M[v] = Op::combine(a, M[v]);
                    }
                }
                if (first < 32) {
                    const int64_t qq = pos - first;
#pragma unroll
                    for (int v = 0; v < CV; ++v) {
                        const float s = (qq >= 0)
                            ? __ldcg(&p.pref[(qq * p.n_chains + chain) * TC + ch + v])
                            : init[v];
                        hin[v] = Op::apply(M[v], s);
                    }
                    break;
                }
                pos -= 32;
            }
            if (timed_out) {
                if (lane == 0) atomicOr(p.status, kTimeoutBit);
#pragma unroll
                for (int v = 0; v < CV; ++v) hin[v] = __int_as_float(0x7fffffff);
            }
        }
        // state entering each warp's rows
        for (int w = 0; w < W; ++w) {
#pragma unroll
            for (int v = 0; v < CV; ++v) s_win[w][ch + v] = Op::apply(s_tot[w][ch + v], hin[v]);
        }
        named_barrier(2, NT);
        if (publish) {
#pragma unroll
            for (int v = 0; v < CV; ++v) __stcg(&p.pref[slot * TC + ch + v], Op::apply(total[v], hin[v]));
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_u64(&p.flags[slot], tag | ST_PREFIX);
        }
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
