// host_pipeline.cu -- scans of tensors that live in host memory
// (mingru_scan_host, minmax_scan_host in include/scan_gated_rnns.h).
//
// The time axis is cut into slices.  Each slice is uploaded on a copy stream,
// scanned on the caller's stream and downloaded on a second copy stream, with
// two sets of device buffers, so PCIe traffic in both directions overlaps the
// scans.  Slice i starts from the last output row of slice i-1, read straight
// from the device buffer that holds it (the scans take an initial state with
// a batch stride), so slicing changes nothing but fp32 rounding order.
// Only the public entry points of the device scans are used here.
#include "scan_gated_rnns.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <limits>
#include <mutex>

namespace {

constexpr size_t kAlign = 256;
// Automatic slicing.  A step costs about the copies in both directions
// (overlapped), plus a fixed cost per slice (measured ~23 us: copy setup,
// events, the scan launch) and the pipeline's fill and drain, which grow
// with the slice (~5 us per MiB of inputs per slice).  The sum is least near
// n = sqrt(input MiB / 4.6) slices: for 256 MiB of inputs (7 slices) a step
// measured 5.67 ms, with 8 slices 5.73 ms, with 33 slices of 8 MB 6.29 ms,
// with 4 slices 5.90 ms and with 64 7.2 ms.
constexpr double kSliceModelMB = 4.6;
constexpr int64_t kMaxAutoSlices = 1024;
constexpr int kMaxDevices = 64;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool mul_ok(int64_t a, int64_t b, int64_t *out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > std::numeric_limits<int64_t>::max() / a) return false;
    *out = a * b;
    return true;
}

// Where everything sits in the caller's staging buffer.
struct Layout {
    int64_t tc = 0;        // rows of T per slice (the last one may be shorter)
    int64_t n = 0;         // slices
    size_t ws = 0;         // scan workspace at offset 0 (status word first)
    size_t off_init = 0;   // (B, D) initial state of slice 0
    size_t off_buf[6] = {};  // slice operands and output, two of each
    size_t total = 0;
};

bool make_layout(sgr_op_t op, int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype, int chunks,
                 Layout *L) {
    const int64_t esz = dtype == SGR_BF16 ? 2 : 4;
    int64_t row = 0, all = 0;     // bytes of one time step of one operand; of both operands
    if (!mul_ok(B, D, &row) || !mul_ok(row, esz, &row) || !mul_ok(row, T, &all) ||
        !mul_ok(all, 2, &all))
        return false;
    int64_t n = chunks;
    if (n <= 0) {
        const double mb = double(all) / double(1 << 20);
        n = std::min<int64_t>(std::max<int64_t>(std::llround(std::sqrt(mb / kSliceModelMB)), 1), kMaxAutoSlices);
    }
    n = std::min<int64_t>(n, T);
    L->tc = (T + n - 1) / n;
    L->n = (T + L->tc - 1) / L->tc;
    const int64_t last = T - (L->n - 1) * L->tc;
    const size_t ws = std::max(sgr_workspace_size(op, B, L->tc, D, dtype),
                               sgr_workspace_size(op, B, last, D, dtype));
    int64_t slice = 0;
    if (!mul_ok(row, L->tc, &slice)) return false;
    L->ws = align_up(std::max<size_t>(ws, kAlign));
    size_t off = L->ws;
    L->off_init = off;
    off += align_up(size_t(row));
    for (int i = 0; i < 6; ++i) {
        L->off_buf[i] = off;
        off += align_up(size_t(slice));
    }
    L->total = off;
    return true;
}

// Library-owned copy streams and the events that order them, one set per
// device, created on first use and kept for the life of the process.  The
// mutex serialises enqueueing, so two host threads never interleave their
// records and waits on the shared events.
struct DeviceQueues {
    std::mutex mu;
    bool ready = false;
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t fork = nullptr, join_up = nullptr, join_down = nullptr;
    cudaEvent_t uploaded[2] = {}, scanned[2] = {}, downloaded[2] = {};
    size_t max_pitch = 0;
};

DeviceQueues g_queues[kMaxDevices];

cudaError_t init_queues(DeviceQueues &q, int dev) {
    cudaError_t e = cudaSuccess;
    auto ev = [&](cudaEvent_t *p) {
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(p, cudaEventDisableTiming);
    };
    e = cudaStreamCreateWithFlags(&q.up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&q.down, cudaStreamNonBlocking);
    ev(&q.fork); ev(&q.join_up); ev(&q.join_down);
    for (int j = 0; j < 2; ++j) { ev(&q.uploaded[j]); ev(&q.scanned[j]); ev(&q.downloaded[j]); }
    int pitch = 0;
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&pitch, cudaDevAttrMaxPitch, dev);
    q.max_pitch = pitch > 0 ? size_t(pitch) : 0;
    return e;
}

// `height` rows of `width` bytes between buffers with the given row pitches.
cudaError_t copy_rows(void *dst, size_t dpitch, const void *src, size_t spitch, size_t width,
                      size_t height, cudaMemcpyKind kind, cudaStream_t s, size_t max_pitch) {
    if (height == 1 || (dpitch == width && spitch == width))
        return cudaMemcpyAsync(dst, src, width * height, kind, s);
    if (dpitch >= width && spitch >= width && dpitch <= max_pitch && spitch <= max_pitch)
        return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, height, kind, s);
    for (size_t r = 0; r < height; ++r) {
        const cudaError_t e = cudaMemcpyAsync(static_cast<char *>(dst) + r * dpitch,
                                              static_cast<const char *>(src) + r * spitch, width,
                                              kind, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// A host buffer: pageable (unregistered) or page-locked memory, not memory of a device.
bool is_host(const void *p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeUnregistered || a.type == cudaMemoryTypeHost;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

}  // namespace

namespace {

sgr_status_t scan_host(sgr_op_t op, const void *in0, const void *in1, const void *init,
                       int64_t init_bs, void *out, int64_t B, int64_t T, int64_t D,
                       sgr_dtype_t dtype, int chunks, void *staging, size_t staging_bytes,
                       cudaStream_t stream) {
    if (dtype != SGR_F32 && dtype != SGR_BF16) return SGR_ERR_INVALID_ARG;
    if (op != SGR_OP_MINGRU && op != SGR_OP_MINMAX) return SGR_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || D < 0 || init_bs < 0 || chunks < 0) return SGR_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || D == 0) return SGR_OK;
    if (!in0 || !in1 || !out) return SGR_ERR_INVALID_ARG;
    const int64_t esz = dtype == SGR_BF16 ? 2 : 4;
    int64_t nbytes = 0, span = 0;
    if (!mul_ok(B, T, &nbytes) || !mul_ok(nbytes, D, &nbytes) || !mul_ok(nbytes, esz, &nbytes))
        return SGR_ERR_UNSUPPORTED;
    if (init && (!mul_ok(B - 1, init_bs, &span) || !mul_ok(span + D, esz, &span)))
        return SGR_ERR_UNSUPPORTED;
    const size_t tb = size_t(nbytes);
    if (overlaps(out, tb, in0, tb) || overlaps(out, tb, in1, tb) ||
        overlaps(out, tb, init, init ? size_t(span) : 0))
        return SGR_ERR_INVALID_ARG;
    if (!is_host(in0) || !is_host(in1) || !is_host(out) || (init && !is_host(init)))
        return SGR_ERR_INVALID_ARG;
    Layout L;
    if (!make_layout(op, B, T, D, dtype, chunks, &L)) return SGR_ERR_UNSUPPORTED;
    if (!staging || staging_bytes < L.total || (reinterpret_cast<uintptr_t>(staging) & 15u))
        return SGR_ERR_WORKSPACE;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return SGR_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return SGR_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SGR_ERR_CUDA;

    DeviceQueues &q = g_queues[dev];
    std::lock_guard<std::mutex> lock(q.mu);
    if (!q.ready) {
        if (init_queues(q, dev) != cudaSuccess) return SGR_ERR_CUDA;
        q.ready = true;
    }
    auto scan = op == SGR_OP_MINGRU ? &mingru_scan : &minmax_scan;
    char *st = static_cast<char *>(staging);
    const char *h0 = static_cast<const char *>(in0), *h1 = static_cast<const char *>(in1);
    char *ho = static_cast<char *>(out);
    const size_t row = size_t(D * esz);          // one (b, t) row of D channels
    const size_t seq = size_t(T) * row;          // one batch row of the host tensors
    const size_t mp = q.max_pitch;
    const auto H2D = cudaMemcpyHostToDevice, D2H = cudaMemcpyDeviceToHost;

    // Fork: both copy streams start after the work already on `stream` (which
    // includes the previous call's use of the staging buffer).
    cudaError_t e = cudaMemsetAsync(st, 0, L.ws, stream);
    if (e == cudaSuccess) e = cudaEventRecord(q.fork, stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(q.up, q.fork, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(q.down, q.fork, 0);
    if (e != cudaSuccess) return SGR_ERR_CUDA;

    sgr_status_t status = SGR_OK;
    const void *dinit = nullptr;
    int64_t dinit_bs = 0;
    if (init) {
        dinit = st + L.off_init;
        if (init_bs == 0 || B == 1) {
            e = cudaMemcpyAsync(st + L.off_init, init, row, H2D, q.up);
        } else {
            e = copy_rows(st + L.off_init, row, init, size_t(init_bs * esz), row, size_t(B), H2D,
                          q.up, mp);
            dinit_bs = D;
        }
        if (e != cudaSuccess) status = SGR_ERR_CUDA;
    }
    for (int64_t i = 0; i < L.n && status == SGR_OK; ++i) {
        const int j = int(i & 1);
        const int64_t t0 = i * L.tc, len = std::min(L.tc, T - t0);
        const size_t w = size_t(len) * row;       // bytes of one batch row of this slice
        char *d0 = st + L.off_buf[j], *d1 = st + L.off_buf[2 + j], *dout = st + L.off_buf[4 + j];
        // upload once the scan two slices back has read this buffer
        if (i >= 2) e = cudaStreamWaitEvent(q.up, q.scanned[j], 0);
        if (e == cudaSuccess) e = copy_rows(d0, w, h0 + t0 * row, seq, w, size_t(B), H2D, q.up, mp);
        if (e == cudaSuccess) e = copy_rows(d1, w, h1 + t0 * row, seq, w, size_t(B), H2D, q.up, mp);
        if (e == cudaSuccess) e = cudaEventRecord(q.uploaded[j], q.up);
        // scan once the slice is in and the download two slices back has left
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, q.uploaded[j], 0);
        if (e == cudaSuccess && i >= 2) e = cudaStreamWaitEvent(stream, q.downloaded[j], 0);
        if (e != cudaSuccess) { status = SGR_ERR_CUDA; break; }
        const void *sinit = dinit;
        int64_t sinit_bs = dinit_bs;
        if (i > 0) {     // the previous slice (full length tc) ends in the other buffer
            sinit = st + L.off_buf[4 + (1 - j)] + size_t(L.tc - 1) * row;
            sinit_bs = L.tc * D;
        }
        status = scan(d0, d1, sinit, sinit_bs, dout, B, len, D, dtype, st, L.ws, stream);
        if (status != SGR_OK) break;
        e = cudaEventRecord(q.scanned[j], stream);
        // download
        if (e == cudaSuccess) e = cudaStreamWaitEvent(q.down, q.scanned[j], 0);
        if (e == cudaSuccess) e = copy_rows(ho + t0 * row, seq, dout, w, w, size_t(B), D2H, q.down, mp);
        if (e == cudaSuccess) e = cudaEventRecord(q.downloaded[j], q.down);
        if (e != cudaSuccess) status = SGR_ERR_CUDA;
    }
    // Join, also after an error: `stream` waits for everything on the copy
    // streams, so later work on it (and the next call) sees them finished.
    bool joined = cudaEventRecord(q.join_up, q.up) == cudaSuccess &&
                  cudaEventRecord(q.join_down, q.down) == cudaSuccess &&
                  cudaStreamWaitEvent(stream, q.join_up, 0) == cudaSuccess &&
                  cudaStreamWaitEvent(stream, q.join_down, 0) == cudaSuccess;
    if (!joined && status == SGR_OK) status = SGR_ERR_CUDA;
    return status;
}

}  // namespace

extern "C" {

size_t sgr_host_staging_size(sgr_op_t op, int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype,
                             int chunks) {
    if (op != SGR_OP_MINGRU && op != SGR_OP_MINMAX) return 0;
    if (dtype != SGR_F32 && dtype != SGR_BF16) return 0;
    if (B <= 0 || T <= 0 || D <= 0 || chunks < 0) return 0;
    Layout L;
    return make_layout(op, B, T, D, dtype, chunks, &L) ? L.total : 0;
}

sgr_status_t mingru_scan_host(const void *k, const void *hx, const void *h0,
                              int64_t h0_batch_stride, void *h, int64_t B, int64_t T, int64_t D,
                              sgr_dtype_t dtype, int chunks, void *staging, size_t staging_bytes,
                              cudaStream_t stream) {
    return scan_host(SGR_OP_MINGRU, k, hx, h0, h0_batch_stride, h, B, T, D, dtype, chunks,
                     staging, staging_bytes, stream);
}

sgr_status_t minmax_scan_host(const void *r, const void *s, const void *x0,
                              int64_t x0_batch_stride, void *x, int64_t B, int64_t T, int64_t D,
                              sgr_dtype_t dtype, int chunks, void *staging, size_t staging_bytes,
                              cudaStream_t stream) {
    return scan_host(SGR_OP_MINMAX, r, s, x0, x0_batch_stride, x, B, T, D, dtype, chunks,
                     staging, staging_bytes, stream);
}

}  // extern "C"
