// q4_gemm_sm100.cu -- q4_gemm for M > 16.
#include "q4_internal.cuh"

namespace q4 {

cudaError_t launch_prefill(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                           const uint16_t* x, float* y, int64_t M, int64_t N, int64_t K,
                           cudaStream_t s, const DeviceInfo& dev) {
    for (int64_t m0 = 0; m0 < M; m0 += 16) {
        const int mc = static_cast<int>(M - m0 < 16 ? M - m0 : 16);
        cudaError_t e = launch_small_m(codes, scales, cb, x + m0 * K, y + m0 * N, mc, N, K, s, dev);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace q4
