// scan_fold.cuh -- slice summaries on TMA-fed warps, sm_100a.
#pragma once

#include "scan_sequential.cuh"

// ------------------------------------------------------- slice summaries
//
// For a time axis split across devices each slice is first reduced to one
// pair per channel: the composition of its steps' pairs (minGRU:
// h_end = A h_start + B; MinMax: x_end = max(min(x_start, U), L)).  Here one
// warp folds one segment of rows of a 32-channel group, through the same
// per-warp ring of TMA boxes as the scans (segments are whole 16-row slots,
// rows past T are skipped), and writes its partial pair; the partials of a
// channel are then folded in segment order (fold_partials_kernel).
namespace sgr {

__host__ __device__ constexpr size_t seq_fold_warp_bytes(int S, int row_bytes) {
    return (size_t(S) * 2 * kSeqRows * row_bytes + size_t(S) * 8 + 127) / 128 * 128;
}

struct SeqFoldParams {
    ScanParams s;        // operands and sizes (no initial state, no output)
    int64_t n_groups;    // channel groups per batch row
    int64_t n_warps;     // n_seg * B * n_groups
    int64_t seg_rows;    // rows per segment, a multiple of the slot height
    int slots;           // load ring depth S
    float2 *partial;     // [n_seg][B][D] pairs
};

template <class Op, typename IO, int WB>
__global__ void __launch_bounds__(WB * 32)
scan_sequential_fold_kernel(const SeqFoldParams q, const __grid_constant__ CUtensorMap map0,
                            const __grid_constant__ CUtensorMap map1) {
    using LR = LaneRow<IO>;
    constexpr int CW = 32;
    constexpr int kRowBytes = seq_row_bytes<IO>();
    constexpr uint32_t kOpBytes = kSeqRows * kRowBytes;
    const ScanParams &p = q.s;
    extern __shared__ __align__(128) unsigned char smem[];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t gw = int64_t(blockIdx.x) * WB + warp;
    if (gw >= q.n_warps) return;                                     // no block barrier below
    const int S = q.slots;
    const int64_t chains = p.B * q.n_groups;
    const int64_t sg = gw / chains;                                  // segment (slowest: chains of a
    const int64_t chain = gw - sg * chains;                          // segment run side by side)
    const int64_t b = chain / q.n_groups;
    const int64_t grp = chain - b * q.n_groups;
    const int x0 = int(grp) * CW;
    const int64_t d = int64_t(x0) + lane;
    const int64_t t0 = sg * q.seg_rows;
    const int64_t t1 = t0 + q.seg_rows < p.T ? t0 + q.seg_rows : p.T;

    const uint32_t ring = smem_addr(smem) + uint32_t(warp * seq_fold_warp_bytes(S, kRowBytes));
    const uint32_t bars = ring + uint32_t(S) * 2 * kOpBytes;
    const int n_slots = int((t1 - t0 + kSeqRows - 1) / kSeqRows);
    auto issue = [&](int i, int s) {
        const uint32_t dst = ring + uint32_t(s) * 2 * kOpBytes;
        const uint32_t bar = bars + 8u * uint32_t(s);
        mbar_expect_tx(bar, 2 * kOpBytes);
        tma_load_3d(dst, &map0, x0, int(t0) + i * kSeqRows, int(b), bar);
        tma_load_3d(dst + kOpBytes, &map1, x0, int(t0) + i * kSeqRows, int(b), bar);
    };
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bars + 8u * s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int s = 0; s < S && s < n_slots; ++s) issue(s, s);
    }
    __syncwarp();

    float2 acc = Op::identity();
    uint32_t wait_limit = kMbarLimit;
    bool bad = false;
    int s = 0;
    uint32_t phase = 0;
    for (int i = 0; i < n_slots; ++i) {
        if (!mbar_wait(bars + 8u * uint32_t(s), phase, wait_limit)) {
            wait_limit = 1;
            if (!bad && lane == 0 && p.status) atomicOr(p.status, kTimeoutBit);
            bad = true;
        }
        const uint32_t src = ring + uint32_t(s) * 2 * kOpBytes + uint32_t(lane) * uint32_t(sizeof(IO));
        float x0r[kSeqRows], x1r[kSeqRows];
#pragma unroll
        for (int r = 0; r < kSeqRows; ++r) {
            x0r[r] = LR::load(src + r * kRowBytes);
            x1r[r] = LR::load(src + kOpBytes + r * kRowBytes);
        }
        __syncwarp();
        if (lane == 0 && !bad && i + S < n_slots) {
            fence_proxy_async();
            issue(i + S, s);
        }
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }
        const int valid = int(t1 - t0 - int64_t(i) * kSeqRows);    // rows of the slot inside the segment
        auto rows = [&](auto fullc) {
            constexpr bool FULL = decltype(fullc)::value;
#pragma unroll
            for (int r = 0; r < kSeqRows; r += 2) {
                float2 a, c;
                Op::element_rows(x0r[r], x1r[r], x0r[r + 1], x1r[r + 1], a, c);
                if (FULL || r < valid) acc = Op::combine(acc, make_float2(a.x, c.x));
                if (FULL || r + 1 < valid) acc = Op::combine(acc, make_float2(a.y, c.y));
            }
        };
        if (valid >= kSeqRows) rows(std::true_type{});
        else rows(std::false_type{});
    }
    if (bad) acc = make_float2(__int_as_float(0x7fffffff), __int_as_float(0x7fffffff));
    if (d < p.D) q.partial[(sg * p.B + b) * p.D + d] = acc;
}

}  // namespace sgr
