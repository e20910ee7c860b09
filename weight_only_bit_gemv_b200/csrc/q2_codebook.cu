// q2_codebook.cu -- the two-bit variant: a 4-entry binary16 codebook, four
// codes per byte, the same 64-weight groups and binary16 scales as the
// four-bit format.  The "Trapetum" overview ("In one sentence", "Frontier
// models on your own hardware") runs a 70B model in 2 bits; the pages print
// no layout, so this one is the four-bit layout with 2-bit codes:
//   codes  [N][K/4]: byte j of row n holds code(n, 4j + i) in bits 2i, 2i+1;
//   scales [N][K/64], codebook [4]: binary16 bit patterns.
//
// pack2 / dequant2: the four-bit steps with four entries, each one IEEE
// operation, so the results are bit-identical to a serial implementation.
//
// gemv2 (one token): one warp owns 16 rows of a "chunk" = 4 groups = 64 code
// bytes per row, and multiplies it with 16 mma.sync m16n8k16 (weights as A,
// fp32 sums).  A chunk's 16 code bytes of one group are one lane's uint4, so
// lane (g, t) (g = lane / 4, t = lane % 4) holds group t of rows g and g + 8.
// The k order inside an MMA is free, because the same permutation is applied
// to x: MMA (q, i) takes, from word q of the lane's uint4, code i of each of
// its four bytes, i.e. k = 16q + i + {0, 4, 8, 12} of the group, as two f16
// pairs built by one PRMT each from the codebook held as split bytes.  The B
// column c carries x of the chunk's group c only (lanes with g == t), so C
// column c is the group's partial sum and is scaled in fp32 by that group's
// scale.  x is staged once per CTA in shared memory as binary16 in the same
// permuted order (8 bytes per MMA and group).  Products are exact (binary16
// times binary16 fits binary32); the chunk sums are fp32.
//
// Work split: the (16-row tile, chunk) pairs of the matrix are one flat list,
// cut into equal contiguous ranges, one per warp; a warp adds each finished
// tile's sums into y with red.add (y is zeroed first on the same stream).
#include "q4_internal.cuh"

namespace q4 {
namespace {

constexpr int kQ2Threads = 256;
constexpr int kQ2Warps = kQ2Threads / 32;
constexpr int kQ2XGroupBytes = 136; // staged x of one group: 16 MMAs x 8 B, + 8 B pad
constexpr int kQ2Batch = 4;         // chunks a warp loads ahead

__device__ __forceinline__ float half_bits_to_float2b(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

__global__ void __launch_bounds__(256) pack2_kernel(const float* __restrict__ w,
                                                    const uint16_t* __restrict__ cb,
                                                    uint8_t* __restrict__ codes,
                                                    uint16_t* __restrict__ scales, int64_t N,
                                                    int64_t K) {
    float c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = half_bits_to_float2b(__ldg(cb + i));
    int zero_code = 0;
    float zero_mag = fabsf(c[0]);
#pragma unroll
    for (int i = 1; i < 4; ++i)
        if (fabsf(c[i]) < zero_mag) {
            zero_mag = fabsf(c[i]);
            zero_code = i;
        }

    const int64_t G = K / kGroup;
    const int64_t total = N * G;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = idx / G, g = idx - n * G;
        const float4* src = reinterpret_cast<const float4*>(w + n * K + g * kGroup);
        float v[kGroup];
#pragma unroll
        for (int q = 0; q < kGroup / 4; ++q) {
            const float4 t = __ldg(src + q);
            v[4 * q + 0] = t.x;
            v[4 * q + 1] = t.y;
            v[4 * q + 2] = t.z;
            v[4 * q + 3] = t.w;
        }
        float a = 0.0f;
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
            const float m = fabsf(v[j]);
            a = (m > a) ? m : a;
        }
        const __half sh = __float2half_rn(a);
        const float s = __half2float(sh);
        uint32_t words[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                int code = zero_code;
                if (s != 0.0f) {
                    const float r = __fdiv_rn(v[16 * q + e], s);
                    code = 0;
                    float best = fabsf(__fsub_rn(r, c[0]));
#pragma unroll
                    for (int i = 1; i < 4; ++i) {
                        const float d = fabsf(__fsub_rn(r, c[i]));
                        if (d < best) {
                            best = d;
                            code = i;
                        }
                    }
                }
                word |= static_cast<uint32_t>(code) << (2 * e);
            }
            words[q] = word;
        }
        *reinterpret_cast<uint4*>(codes + n * (K / 4) + g * (kGroup / 4)) =
            make_uint4(words[0], words[1], words[2], words[3]);
        scales[n * G + g] = __half_as_ushort(sh);
    }
}

// One thread rebuilds 16 consecutive weights of one row (one code word).
__global__ void __launch_bounds__(256) dequant2_kernel(const uint8_t* __restrict__ codes,
                                                       const uint16_t* __restrict__ scales,
                                                       const uint16_t* __restrict__ cb,
                                                       float* __restrict__ w, int64_t N,
                                                       int64_t K) {
    float c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = half_bits_to_float2b(__ldg(cb + i));
    const int64_t per_row = K / 16;
    const int64_t total = N * per_row;
    const int64_t G = K / kGroup;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = idx / per_row, j = idx - n * per_row;
        const int64_t k0 = j * 16;
        const uint32_t word = __ldg(reinterpret_cast<const uint32_t*>(codes + n * (K / 4) + j * 4));
        const float s = half_bits_to_float2b(scales[n * G + k0 / kGroup]);
        float out[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint32_t code = (word >> (2 * e)) & 3u;
            const float v = (code & 2u) ? ((code & 1u) ? c[3] : c[2]) : ((code & 1u) ? c[1] : c[0]);
            out[e] = __fmul_rn(v, s);
        }
        float4* dst = reinterpret_cast<float4*>(w + n * K + k0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            dst[q] = make_float4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
    }
}

int grid_for2(int64_t items, int threads, const DeviceInfo& dev) {
    const int64_t blocks = (items + threads - 1) / threads;
    const int64_t cap = static_cast<int64_t>(dev.sm_count) * 16;
    return static_cast<int>(blocks < cap ? blocks : cap);
}

// The code bytes of one lane for one chunk: group t of rows g and g + 8, and
// the two scales.  Zeros where the row or the group does not exist (the B
// column of a missing group is zero, so its A values never count).
struct Q2Chunk {
    uint4 wa, wb;
    uint16_t sa, sb;
};

__device__ __forceinline__ Q2Chunk load_chunk2(const uint8_t* __restrict__ codes,
                                               const uint16_t* __restrict__ scales, int64_t f,
                                               int64_t f_end, int64_t CH, int64_t N, int64_t K,
                                               int64_t G, int g, int t) {
    Q2Chunk c;
    c.wa = make_uint4(0u, 0u, 0u, 0u);
    c.wb = c.wa;
    c.sa = 0;
    c.sb = 0;
    if (f < f_end) {
        const int64_t rt = f / CH, ch = f - rt * CH;
        const int64_t grp = 4 * ch + t;
        const int64_t ra = 16 * rt + g, rb = ra + 8;
        if (grp < G) {
            if (ra < N) {
                c.wa = __ldcs(reinterpret_cast<const uint4*>(codes + ra * (K / 4) + grp * 16));
                c.sa = __ldg(reinterpret_cast<const unsigned short*>(scales + ra * G + grp));
            }
            if (rb < N) {
                c.wb = __ldcs(reinterpret_cast<const uint4*>(codes + rb * (K / 4) + grp * 16));
                c.sb = __ldg(reinterpret_cast<const unsigned short*>(scales + rb * G + grp));
            }
        }
    }
    return c;
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int q) {
    return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}

__global__ void __launch_bounds__(kQ2Threads, 2)
    gemv2_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                 const uint16_t* __restrict__ cb, const uint16_t* __restrict__ x,
                 float* __restrict__ y, int64_t N, int64_t K) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int64_t G = K / kGroup;

    // x as binary16 in MMA order: group G at G * 136, MMA (q, i) at 8 * (4q + i),
    // holding k = 16q + i + {0, 4, 8, 12} of the group
    for (int64_t k = threadIdx.x; k < K; k += blockDim.x) {
        const int64_t grp = k / kGroup;
        const int r = static_cast<int>(k - grp * kGroup);
        const int q = r >> 4, j = (r >> 2) & 3, i = r & 3;
        const __half h = __float2half_rn(bf16_bits_to_float(__ldg(x + k)));
        *reinterpret_cast<__half*>(smem + grp * kQ2XGroupBytes + 8 * (4 * q + i) + 2 * j) = h;
    }
    __syncthreads();

    // codebook split into its low bytes (lo) and high bytes (hi): PRMT index
    // c picks entry c's low byte, 4 + c its high byte
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t h = __ldg(cb + e);
        lo |= (h & 0xFFu) << (8 * e);
        hi |= (h >> 8) << (8 * e);
    }

    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const bool xlane = (g == t);
    const int64_t CH = (G + 3) / 4;
    const int64_t RT = (N + 15) / 16;
    const int64_t F = RT * CH;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * kQ2Warps;
    const int64_t wid = static_cast<int64_t>(blockIdx.x) * kQ2Warps + (threadIdx.x >> 5);
    const int64_t f_begin = wid * F / warps, f_end = (wid + 1) * F / warps;

    float part_a = 0.f, part_b = 0.f;  // rows g and g + 8 of the current tile
    int64_t cur_rt = -1;
    auto flush = [&](int64_t rt) {
        float va = part_a + __shfl_xor_sync(0xFFFFFFFFu, part_a, 1);
        float vb = part_b + __shfl_xor_sync(0xFFFFFFFFu, part_b, 1);
        if (rt >= 0 && t == 0) {
            const int64_t ra = 16 * rt + g, rb = ra + 8;
            if (ra < N) atomicAdd(y + ra, va);
            if (rb < N) atomicAdd(y + rb, vb);
        }
        part_a = 0.f;
        part_b = 0.f;
    };

    Q2Chunk cur[kQ2Batch];
#pragma unroll
    for (int u = 0; u < kQ2Batch; ++u)
        cur[u] = load_chunk2(codes, scales, f_begin + u, f_end, CH, N, K, G, g, t);

    for (int64_t f = f_begin; f < f_end; f += kQ2Batch) {
        Q2Chunk nxt[kQ2Batch];
#pragma unroll
        for (int u = 0; u < kQ2Batch; ++u)
            nxt[u] = load_chunk2(codes, scales, f + kQ2Batch + u, f_end, CH, N, K, G, g, t);

#pragma unroll
        for (int u = 0; u < kQ2Batch; ++u) {
            const int64_t ff = f + u;
            if (ff < f_end) {  // warp-uniform
                const int64_t rt = ff / CH, ch = ff - rt * CH;
                if (rt != cur_rt) {
                    flush(cur_rt);
                    cur_rt = rt;
                }
                const int64_t grp = 4 * ch + t;
                const bool xon = xlane && grp < G;
                const uint8_t* xg = smem + (xon ? grp : 0) * kQ2XGroupBytes;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t wa = word_of(cur[u].wa, q), wb = word_of(cur[u].wb, q);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t sel_a = ((wa >> (2 * i)) & 0x03030303u) * 0x11u + 0x40404040u;
                        const uint32_t sel_b = ((wb >> (2 * i)) & 0x03030303u) * 0x11u + 0x40404040u;
                        uint32_t a[4];
                        a[0] = __byte_perm(lo, hi, sel_a);        // row g,     k +0, +4
                        a[1] = __byte_perm(lo, hi, sel_b);        // row g + 8, k +0, +4
                        a[2] = __byte_perm(lo, hi, sel_a >> 16);  // row g,     k +8, +12
                        a[3] = __byte_perm(lo, hi, sel_b >> 16);  // row g + 8, k +8, +12
                        uint2 xb = make_uint2(0u, 0u);
                        if (xon) xb = ld_smem<uint2>(xg, 8 * (4 * q + i));
                        mma_16816(acc, a, xb.x, xb.y, acc);
                    }
                }
                // C columns 2t, 2t + 1 are groups 4ch + 2t, + 1; their scales
                // sit in lanes (g, 2t) and (g, 2t + 1).  Lanes t >= 2 hold
                // the zero columns 4..7.
                const int src0 = (lane & ~3) | ((2 * t) & 3), src1 = (lane & ~3) | ((2 * t + 1) & 3);
                const float sa0 = half_bits_to_float2b(__shfl_sync(0xFFFFFFFFu, cur[u].sa, src0));
                const float sa1 = half_bits_to_float2b(__shfl_sync(0xFFFFFFFFu, cur[u].sa, src1));
                const float sb0 = half_bits_to_float2b(__shfl_sync(0xFFFFFFFFu, cur[u].sb, src0));
                const float sb1 = half_bits_to_float2b(__shfl_sync(0xFFFFFFFFu, cur[u].sb, src1));
                if (t < 2) {
                    part_a = fmaf(acc[0], sa0, fmaf(acc[1], sa1, part_a));
                    part_b = fmaf(acc[2], sb0, fmaf(acc[3], sb1, part_b));
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kQ2Batch; ++u) cur[u] = nxt[u];
    }
    flush(cur_rt);
}

}  // namespace

cudaError_t launch_pack2(const float* w, const uint16_t* cb, uint8_t* codes, uint16_t* scales,
                         int64_t N, int64_t K, cudaStream_t s, const DeviceInfo& dev) {
    const int64_t groups = N * (K / kGroup);
    pack2_kernel<<<grid_for2(groups, 256, dev), 256, 0, s>>>(w, cb, codes, scales, N, K);
    return cudaGetLastError();
}

cudaError_t launch_dequant2(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                            float* w, int64_t N, int64_t K, cudaStream_t s, const DeviceInfo& dev) {
    const int64_t items = N * (K / 16);
    dequant2_kernel<<<grid_for2(items, 256, dev), 256, 0, s>>>(codes, scales, cb, w, N, K);
    return cudaGetLastError();
}

int gemv2_smem_bytes(int64_t K) { return static_cast<int>((K / kGroup) * kQ2XGroupBytes); }

cudaError_t launch_gemv2(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                         const uint16_t* x, float* y, int64_t N, int64_t K, cudaStream_t s,
                         const DeviceInfo& dev) {
    const int smem = gemv2_smem_bytes(K);
    if (smem > dev.smem_optin) return cudaErrorNotSupported;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(gemv2_kernel), smem, 50, dev.device);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(y, 0, static_cast<size_t>(N) * sizeof(float), s);
    if (e != cudaSuccess) return e;
    // two CTAs per SM when both fit beside the per-CTA reservation
    const int per_sm = (2 * (smem + dev.smem_reserved) <= 228 * 1024) ? 2 : 1;
    gemv2_kernel<<<dev.sm_count * per_sm, kQ2Threads, smem, s>>>(codes, scales, cb, x, y, N, K);
    return cudaGetLastError();
}

}  // namespace q4
