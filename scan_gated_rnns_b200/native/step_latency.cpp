// step_latency -- token-by-token decoding through the C ABI, timed from a
// plain host loop (no Python, no CUDA graph): the per-token cost a C or C++
// caller of mingru_step pays (page "Mingru Pytorch", guide "Process a
// sequence sequentially with carried hidden state": one call per token with
// the state carried between calls; page "MinMax Recurrent Neural Cascades",
// Key properties: O(1) work per token).
//
//   step_latency B D steps warmup
//
// Runs `warmup` then `steps` calls of mingru_step on (B, D) fp32 rows, the
// state updated in place on one stream, and prints one JSON line:
//   us_per_call_host   host time to issue one call (argument checks + launch)
//   us_per_step_device device time per step with the calls back to back
//                      (CUDA events around the timed calls on the stream)
//   us_per_step_wall   host time per step from the first call to the end of
//                      the last step (issue-bound or device-bound, whichever
//                      is slower)
// Inputs come from a fixed linear congruential generator, uniform in
// [-2, 2) for k and hx, the state starting at 0.5.
#include "scan_gated_rnns.h"

#include <cuda_runtime.h>

#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <vector>

namespace {

bool ok(cudaError_t e, const char *what) {
    if (e != cudaSuccess) {
        std::fprintf(stderr, "step_latency: %s: %s\n", what, cudaGetErrorString(e));
        return false;
    }
    return true;
}

double now_us() {
    using clk = std::chrono::steady_clock;
    return std::chrono::duration<double, std::micro>(clk::now().time_since_epoch()).count();
}

}  // namespace

int main(int argc, char **argv) {
    const long long B = argc > 1 ? std::atoll(argv[1]) : 8;
    const long long D = argc > 2 ? std::atoll(argv[2]) : 1024;
    const int steps = argc > 3 ? std::atoi(argv[3]) : 2000;
    const int warmup = argc > 4 ? std::atoi(argv[4]) : 100;
    if (B <= 0 || D <= 0 || steps <= 0 || warmup < 0) {
        std::fprintf(stderr, "usage: step_latency B D steps warmup\n");
        return 2;
    }
    const size_t n = size_t(B) * size_t(D);
    std::vector<float> host(3 * n);
    uint64_t s = 0x9e3779b97f4a7c15ull;
    for (size_t i = 0; i < 2 * n; ++i) {
        s = s * 6364136223846793005ull + 1442695040888963407ull;
        host[i] = float(double(s >> 40) / double(1ull << 24) * 4.0 - 2.0);
    }
    for (size_t i = 2 * n; i < 3 * n; ++i) host[i] = 0.5f;
    float *dev = nullptr;
    if (!ok(cudaMalloc(&dev, 3 * n * sizeof(float)), "cudaMalloc")) return 1;
    cudaStream_t st = nullptr;
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    int rc = 1;
    do {
        if (!ok(cudaMemcpy(dev, host.data(), 3 * n * sizeof(float), cudaMemcpyHostToDevice), "copy in")) break;
        if (!ok(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking), "stream")) break;
        if (!ok(cudaEventCreate(&e0), "event") || !ok(cudaEventCreate(&e1), "event")) break;
        const float *k = dev, *hx = dev + n;
        float *h = dev + 2 * n;
        auto step = [&]() {
            return mingru_step(k, D, hx, D, h, D, h, D, B, D, SGR_F32, st);
        };
        sgr_status_t status = SGR_OK;
        for (int i = 0; i < warmup && status == SGR_OK; ++i) status = step();
        if (status != SGR_OK || !ok(cudaStreamSynchronize(st), "warm-up")) {
            std::fprintf(stderr, "step_latency: %s\n", sgr_status_string(status));
            break;
        }
        const double t0 = now_us();
        if (!ok(cudaEventRecord(e0, st), "record")) break;
        for (int i = 0; i < steps && status == SGR_OK; ++i) status = step();
        const double t1 = now_us();
        if (status != SGR_OK) {
            std::fprintf(stderr, "step_latency: %s\n", sgr_status_string(status));
            break;
        }
        if (!ok(cudaEventRecord(e1, st), "record") || !ok(cudaEventSynchronize(e1), "sync")) break;
        const double t2 = now_us();
        float ms = 0.f;
        if (!ok(cudaEventElapsedTime(&ms, e0, e1), "elapsed")) break;
        std::printf("{\"B\": %lld, \"D\": %lld, \"steps\": %d, \"us_per_call_host\": %.3f, "
                    "\"us_per_step_device\": %.3f, \"us_per_step_wall\": %.3f}\n",
                    B, D, steps, (t1 - t0) / steps, double(ms) * 1e3 / steps, (t2 - t0) / steps);
        rc = 0;
    } while (false);
    if (e0) cudaEventDestroy(e0);
    if (e1) cudaEventDestroy(e1);
    if (st) cudaStreamDestroy(st);
    cudaFree(dev);
    return rc;
}
