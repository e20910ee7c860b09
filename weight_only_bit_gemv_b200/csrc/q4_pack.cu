// q4_pack.cu -- pack (quantize) and dequantize kernels.
//
// Pack follows the group format of the "deep-fold" page, section "Method":
// 64 weights per group, four-bit codes into a 16-entry codebook and one FP16
// scale.  Per group: scale = binary16(absmax) rounded to nearest-even; code =
// the codebook index nearest to w / scale, with the division and the
// distances in IEEE binary32 and ties to the lowest index; a zero scale maps
// every weight to the entry of smallest magnitude.  Each step is one IEEE
// operation (__fdiv_rn, __fsub_rn, cvt.rn.f16.f32), so the result is
// bit-identical to any serial IEEE implementation of the same steps.
//
// Dequant writes W = codebook[code] * scale in binary32, which is exact.
// Embed-rows writes the same values for the requested rows only ("deep-fold",
// introduction and Figure 1: embeddings decode only the requested rows, on a
// path of their own).
#include "q4_internal.cuh"

namespace q4 {
namespace {

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

__global__ void __launch_bounds__(256) pack_kernel(const float* __restrict__ w,
                                                   const uint16_t* __restrict__ cb,
                                                   uint8_t* __restrict__ codes,
                                                   uint16_t* __restrict__ scales, int64_t N,
                                                   int64_t K) {
    __shared__ float cbf[16];
    __shared__ int zero_code_s;
    if (threadIdx.x < 16) cbf[threadIdx.x] = half_bits_to_float(cb[threadIdx.x]);
    __syncthreads();
    if (threadIdx.x == 0) {
        int z = 0;
        for (int i = 1; i < 16; ++i)
            if (fabsf(cbf[i]) < fabsf(cbf[z])) z = i;
        zero_code_s = z;
    }
    __syncthreads();
    float c[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) c[i] = cbf[i];
    const int zero_code = zero_code_s;

    const int64_t G = K / kGroup;
    const int64_t total = N * G;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = idx / G, g = idx - n * G;
        if (!Q4_IN_BOUNDS(n * K + g * kGroup, kGroup, N * K) ||
            !Q4_IN_BOUNDS(n * (K / 2) + g * (kGroup / 2), kGroup / 2, N * (K / 2)) ||
            !Q4_IN_BOUNDS(n * G + g, 1, N * G))
            continue;
        const float4* src = reinterpret_cast<const float4*>(w + n * K + g * kGroup);
        float v[kGroup];
#pragma unroll
        for (int q = 0; q < kGroup / 4; ++q) {
            float4 t = __ldg(src + q);
            v[4 * q + 0] = t.x;
            v[4 * q + 1] = t.y;
            v[4 * q + 2] = t.z;
            v[4 * q + 3] = t.w;
        }
        float a = 0.0f;
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
            float m = fabsf(v[j]);
            a = (m > a) ? m : a;
        }
        const __half sh = __float2half_rn(a);
        const float s = __half2float(sh);
        uint32_t words[kGroup / 8];
#pragma unroll
        for (int q = 0; q < kGroup / 8; ++q) {
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                int code = zero_code;
                if (s != 0.0f) {
                    const float r = __fdiv_rn(v[8 * q + e], s);
                    code = 0;
                    float best = fabsf(__fsub_rn(r, c[0]));
#pragma unroll
                    for (int i = 1; i < 16; ++i) {
                        const float d = fabsf(__fsub_rn(r, c[i]));
                        if (d < best) {
                            best = d;
                            code = i;
                        }
                    }
                }
                word |= static_cast<uint32_t>(code) << (4 * e);
            }
            words[q] = word;
        }
        uint4* dst = reinterpret_cast<uint4*>(codes + n * (K / 2) + g * (kGroup / 2));
        dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
        dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
        scales[n * G + g] = __half_as_ushort(sh);
    }
}

// One thread rebuilds 16 consecutive weights of one row (8 code bytes).
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ codes,
                                                      const uint16_t* __restrict__ scales,
                                                      const uint16_t* __restrict__ cb,
                                                      float* __restrict__ w, int64_t N,
                                                      int64_t K) {
    __shared__ float cbf[16];
    if (threadIdx.x < 16) cbf[threadIdx.x] = half_bits_to_float(cb[threadIdx.x]);
    __syncthreads();
    const int64_t per_row = K / 16;
    const int64_t total = N * per_row;
    const int64_t G = K / kGroup;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = idx / per_row, j = idx - n * per_row;
        const int64_t k0 = j * 16;
        if (!Q4_IN_BOUNDS(n * (K / 2) + j * 8, 8, N * (K / 2)) || !Q4_IN_BOUNDS(n * G + k0 / kGroup, 1, N * G) ||
            !Q4_IN_BOUNDS(n * K + k0, 16, N * K))
            continue;
        const uint2 b = __ldg(reinterpret_cast<const uint2*>(codes + n * (K / 2) + j * 8));
        const float s = half_bits_to_float(scales[n * G + k0 / kGroup]);
        float out[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t word = (e < 4) ? b.x : b.y;
            const uint32_t code = (word >> (4 * (e % 4) * 2)) & 0xFFu;
            out[2 * e] = __fmul_rn(cbf[code & 0xF], s);
            out[2 * e + 1] = __fmul_rn(cbf[code >> 4], s);
        }
        float4* dst = reinterpret_cast<float4*>(w + n * K + k0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            dst[q] = make_float4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
    }
}

int grid_for(int64_t items, int threads, const DeviceInfo& dev) {
    int64_t blocks = (items + threads - 1) / threads;
    int64_t cap = static_cast<int64_t>(dev.sm_count) * 16;
    return static_cast<int>(blocks < cap ? blocks : cap);
}

}  // namespace

cudaError_t launch_pack(const float* w, const uint16_t* cb, uint8_t* codes, uint16_t* scales,
                        int64_t N, int64_t K, cudaStream_t s, const DeviceInfo& dev) {
    const int64_t groups = N * (K / kGroup);
    pack_kernel<<<grid_for(groups, 256, dev), 256, 0, s>>>(w, cb, codes, scales, N, K);
    return cudaGetLastError();
}

// Row ids[i] of the packed matrix, dequantized into out[i]; ids outside
// [0, N) give a row of zeros.  A thread writes 16 consecutive values (one
// 8-byte code load, four 16-byte stores), so a warp's stores are contiguous.
__global__ void __launch_bounds__(256) embed_rows_kernel(const uint8_t* __restrict__ codes,
                                                         const uint16_t* __restrict__ scales,
                                                         const uint16_t* __restrict__ cb,
                                                         const int32_t* __restrict__ ids,
                                                         float* __restrict__ out, int64_t n_ids,
                                                         int64_t N, int64_t K) {
    __shared__ float cbf[16];
    if (threadIdx.x < 16) cbf[threadIdx.x] = half_bits_to_float(cb[threadIdx.x]);
    __syncthreads();
    const int64_t per_row = K / 16;
    const int64_t total = n_ids * per_row;
    const int64_t G = K / kGroup;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = idx / per_row, j = idx - i * per_row;
        const int64_t k0 = j * 16;
        if (!Q4_IN_BOUNDS(i, 1, n_ids) || !Q4_IN_BOUNDS(i * K + k0, 16, n_ids * K)) continue;
        const int64_t n = __ldg(ids + i);
        float v[16];
        if (n >= 0 && n < N && Q4_IN_BOUNDS(n * (K / 2) + j * 8, 8, N * (K / 2)) &&
            Q4_IN_BOUNDS(n * G + k0 / kGroup, 1, N * G)) {
            const uint2 b = __ldg(reinterpret_cast<const uint2*>(codes + n * (K / 2) + j * 8));
            const float sc = half_bits_to_float(scales[n * G + k0 / kGroup]);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t word = (e < 4) ? b.x : b.y;
                const uint32_t code = (word >> (8 * (e % 4))) & 0xFFu;
                v[2 * e] = __fmul_rn(cbf[code & 0xF], sc);
                v[2 * e + 1] = __fmul_rn(cbf[code >> 4], sc);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0.f;
        }
        float4* dst = reinterpret_cast<float4*>(out + i * K + k0);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
}

cudaError_t launch_dequant(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                           float* w, int64_t N, int64_t K, cudaStream_t s, const DeviceInfo& dev) {
    const int64_t items = N * (K / 16);
    dequant_kernel<<<grid_for(items, 256, dev), 256, 0, s>>>(codes, scales, cb, w, N, K);
    return cudaGetLastError();
}

cudaError_t launch_embed_rows(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                             const int32_t* ids, float* out, int64_t n_ids, int64_t N, int64_t K,
                             cudaStream_t s, const DeviceInfo& dev) {
    const int64_t items = n_ids * (K / 16);
    embed_rows_kernel<<<grid_for(items, 256, dev), 256, 0, s>>>(codes, scales, cb, ids, out, n_ids, N,
                                                               K);
    return cudaGetLastError();
}

Q4_DEFINE_TAKE_BOUNDS(pack)

}  // namespace q4
