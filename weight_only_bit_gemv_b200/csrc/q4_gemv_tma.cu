// q4_gemv_tma.cu -- the M = 1 decode GEMV on sm_100a: a warp-specialized TMA
// pipeline over the canonical row-major code layout.
//
// What it computes: y[n] = sum_g scale[n][g] * sum_{k in g} cb[code(n,k)] * x[k]
// ("deep-fold", "Method": 64-weight groups, four-bit codes, one FP16 scale;
// the decode GEMV rebuilds values while it multiplies; "Trapetum" overview,
// "The bandwidth law": decode time is set by the weight bytes read).
//
// Why this shape.  Decode streams 0.53125 bytes per weight; at the HBM rate
// every SM must retire ~40 weights per clock.  Decoding a weight costs 2
// bytes of shared-memory bandwidth (one 4-byte table read per code byte), so
// all other traffic through the SM's load/store pipe is kept small:
//  * codes arrive by TMA: per stage two boxes of 128 rows x 128 bytes (8
//    groups of 64 weights), instead of per-lane global loads that would touch
//    eight cache lines per warp instruction;
//  * scales arrive by TMA too (a box of 128 rows x 8 scales) when the row
//    stride of the scale matrix is a multiple of 16 bytes, else by cp.async;
//  * x is bulk-copied once per CTA, rounded to binary16 in shared memory.
// One producer warp fills an S-stage ring; 8 consumer warps each own 16 rows
// of the 128-row strip.  Consumer lane (g, tq) reads rows 2g and 2g+1 of its
// warp's 16; with the 128-byte swizzle of the boxes every 8-byte shared load
// of codes is conflict-free.
//
// Decode and multiply: each code byte indexes a 256-entry byte -> half2 table
// (cb[lo nibble], cb[hi nibble]) replicated once per lane (entry b of lane l
// at byte 256 b + 4 l), so a PRMT builds the address and one LDS returns two
// weights.  The binary16 weights are the A operand of mma.sync m16n8k16, x is
// the B operand; binary16 products are exact and accumulate in fp32.  One
// MMA chain covers one 64-weight group, so the group's fp32 sum is scaled by
// the group's scale in fp32.  Only column 0 of B (lanes 0-3) carries x.
//
// Work split: CTAs are persistent, one per SM, and take equal contiguous
// ranges of (strip, k-stage) units.  A strip covered by one CTA is stored;
// a strip shared between CTAs is accumulated with red.add into y, which the
// host zeroes first.
//
// Start-up: x and the codebook are copied first; the weight stream starts
// only after the table is built, because requests queued behind the weight
// stream of all SMs wait microseconds.
#include "q4_internal.cuh"
#include "q4_sm100.cuh"

namespace q4 {

__device__ unsigned int g_gemv_tma_error;

namespace {

// Consumer warps: kTiles 16-row tiles x kHalves.  With two halves, warp
// (tile, h) decodes groups 4h .. 4h+3 of every stage (one code box each) and
// the two halves of a tile add up at the end of a strip; measured on B200 it
// is no faster than one warp per tile, which is the setting used.
constexpr int kTiles = 8;
constexpr int kHalves = 1;
constexpr int kC = kTiles * kHalves;         // consumer warps
constexpr int kR = 16 * kTiles;              // rows per strip
constexpr int kSG = 8;                       // groups per stage
constexpr int kBoxBytes = kR * 128;          // one code box: 4 groups x 128 rows
constexpr int kCodeStageBytes = 2 * kBoxBytes;
constexpr int kScaleStageBytes = kR * kSG * 2;
constexpr int kLutBytes = 65536;
constexpr int kThreads = (kC + 1) * 32;
constexpr int kMaxStages = 6;

enum ScaleMode { kScaleTma = 0, kScaleAsync = 1, kScaleSync = 2 };

struct TmaGemv {
    const uint16_t* scales;
    const uint16_t* cb;
    const uint16_t* x;
    float* y;
    int N, K, G, KS, strips;
    int stages;
    int scale_off, xs_off, cb_off, pair_off, bar_off;
};

__device__ __forceinline__ uint32_t cvt_bf16x2_f16x2(uint32_t w) {
    const __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float half_lo(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<uint16_t>(w & 0xFFFFu)));
}
__device__ __forceinline__ float half_hi(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<uint16_t>(w >> 16)));
}

// Table entry (cb[lo], cb[hi]) for byte kByte of `word`, this lane's copy:
// offset [lane*4, code byte, 0, 0].
template <int kByte>
__device__ __forceinline__ uint32_t lut_at(const uint8_t* smem, uint32_t word, uint32_t lane4) {
    return ld_smem<uint32_t>(smem, __byte_perm(word, lane4, 0x5504 | (kByte << 4)));
}

// Lane 0 polls, the warp follows.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int lane) {
    uint32_t ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity) ? 1u : 0u;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    __syncwarp();  // orders lane 0's acquire before the other lanes' accesses
    return ok != 0;
}

// One 64-weight group of the two rows this lane decodes: four chained MMAs
// over the group's 64 k.  Returns column 0 of rows g and g + 8.
__device__ __forceinline__ void group_mma(const uint8_t* smem, uint2 lo, uint2 hi, uint4 x0,
                                          uint4 x1, uint32_t lane4, float& d0, float& d2) {
    const float z[4] = {0.f, 0.f, 0.f, 0.f};
    float d[4];
    uint32_t a[4];
    a[0] = lut_at<0>(smem, lo.x, lane4);
    a[1] = lut_at<0>(smem, hi.x, lane4);
    a[2] = lut_at<1>(smem, lo.x, lane4);
    a[3] = lut_at<1>(smem, hi.x, lane4);
    mma_16816(d, a, x0.x, x0.y, z);
    a[0] = lut_at<2>(smem, lo.x, lane4);
    a[1] = lut_at<2>(smem, hi.x, lane4);
    a[2] = lut_at<3>(smem, lo.x, lane4);
    a[3] = lut_at<3>(smem, hi.x, lane4);
    mma_16816(d, a, x0.z, x0.w, d);
    a[0] = lut_at<0>(smem, lo.y, lane4);
    a[1] = lut_at<0>(smem, hi.y, lane4);
    a[2] = lut_at<1>(smem, lo.y, lane4);
    a[3] = lut_at<1>(smem, hi.y, lane4);
    mma_16816(d, a, x1.x, x1.y, d);
    a[0] = lut_at<2>(smem, lo.y, lane4);
    a[1] = lut_at<2>(smem, hi.y, lane4);
    a[2] = lut_at<3>(smem, lo.y, lane4);
    a[3] = lut_at<3>(smem, hi.y, lane4);
    mma_16816(d, a, x1.z, x1.w, d);
    d0 = d[0];
    d2 = d[2];
}

template <int kScale>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_tma_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap smap,
                    const TmaGemv p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t base = smem_u32(smem);
    const uint32_t bars = base + p.bar_off;
    const int S = p.stages;
    auto full = [&](int s) { return bars + 8u * s; };
    auto empty = [&](int s) { return bars + 8u * (S + s); };
    const uint32_t xbar = bars + 16u * S;  // x and codebook landed

    const long long U = static_cast<long long>(p.strips) * p.KS;
    const long long u0 = U * blockIdx.x / gridDim.x;
    const long long u1 = U * (blockIdx.x + 1) / gridDim.x;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            // TMA scales: the expect_tx arrival alone; otherwise one more per lane
            mbar_init(full(s), kScale == kScaleTma ? 1 : 33);
            mbar_init(empty(s), kC);  // one arrival per consumer warp
        }
        mbar_init(xbar, 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kC) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tensor_map(&tmap);
            if (kScale == kScaleTma) prefetch_tensor_map(&smap);
            mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(p.K) * 2u + 32u);
            bulk_load(base + p.xs_off, p.x, static_cast<uint32_t>(p.K) * 2u, xbar);
            bulk_load(base + p.cb_off, p.cb, 32u, xbar);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");  // table and x ready

        int slot = 0, round = 0;
        long long u = u0;
        int strip = static_cast<int>(u / p.KS), ks = static_cast<int>(u % p.KS);
        for (; u < u1; ++u) {
            // reuse of a slot waits for the consumers' release of round - 1
            if (round > 0 && !warp_wait(empty(slot), static_cast<uint32_t>(round + 1) & 1u, lane)) {
                if (lane == 0) atomicOr(&g_gemv_tma_error, 1u);
                return;
            }
            const uint32_t cdst = base + kLutBytes + slot * kCodeStageBytes;
            const uint32_t sdst = base + p.scale_off + slot * kScaleStageBytes;
            if (lane == 0) {
                mbar_arrive_expect_tx(full(slot), kCodeStageBytes +
                                                      (kScale == kScaleTma ? kScaleStageBytes : 0));
                tma_load_2d(cdst, &tmap, ks * 256, strip * kR, full(slot));
                tma_load_2d(cdst + kBoxBytes, &tmap, ks * 256 + 128, strip * kR, full(slot));
                if (kScale == kScaleTma) tma_load_2d(sdst, &smap, ks * kSG, strip * kR, full(slot));
            }
            if (kScale != kScaleTma) {
#pragma unroll
                for (int j = 0; j < kR / 32; ++j) {
                    const int r = lane + 32 * j;
                    const int row = strip * kR + r;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int g0 = ks * kSG + 4 * h;
                        if (kScale == kScaleAsync) {
                            const bool ok = row < p.N && g0 < p.G;
                            const uint16_t* src =
                                ok ? p.scales + static_cast<long long>(row) * p.G + g0 : p.scales;
                            cp_async_8(sdst + r * 16 + 8 * h, src, ok ? 8u : 0u);
                        } else {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                uint16_t v = 0;
                                if (row < p.N && g0 + q < p.G)
                                    v = p.scales[static_cast<long long>(row) * p.G + g0 + q];
                                sts_u16(sdst + r * 16 + 8 * h + 2 * q, v);
                            }
                        }
                    }
                }
                if (kScale == kScaleAsync)
                    cp_async_arrive_noinc(full(slot));
                else
                    mbar_arrive(full(slot));
            }
            if (++slot == S) {
                slot = 0;
                ++round;
            }
            if (++ks == p.KS) {
                ks = 0;
                ++strip;
            }
        }
        // Leave only once the copies this warp issued have landed (bounded).
        const long long n = u1 - u0;
        for (long long i = (n > S ? n - S : 0); i < n; ++i) {
            const int sl = static_cast<int>(i % S);
            if (!warp_wait(full(sl), static_cast<uint32_t>(i / S) & 1u, lane)) {
                if (lane == 0) atomicOr(&g_gemv_tma_error, 4u);
                break;
            }
        }
        return;
    }

    // ------------------------------- consumers ------------------------------
    // Wait for x and the codebook, build the byte -> (cb[lo], cb[hi]) table
    // (one copy per lane) and round x to binary16 in place, zero-padded to
    // whole stages.
    {
        if (!warp_wait(xbar, 0u, lane)) {
            if (lane == 0) atomicOr(&g_gemv_tma_error, 8u);
            asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
            return;
        }
        const uint32_t cbv = ld_smem<uint16_t>(smem, p.cb_off + 2 * (lane & 15));
        for (int b = warp; b < 256; b += kC) {
            const uint32_t lo = __shfl_sync(0xFFFFFFFFu, cbv, b & 15);
            const uint32_t hi = __shfl_sync(0xFFFFFFFFu, cbv, b >> 4);
            *reinterpret_cast<uint32_t*>(smem + b * 256 + lane * 4) = lo | (hi << 16);
        }
        const int units = p.KS * kSG * kGroup / 8;
        for (int i = tid; i < units; i += kC * 32) {
            uint4 h = make_uint4(0u, 0u, 0u, 0u);
            if (i * 8 < p.K) {
                const uint4 v = ld_smem<uint4>(smem, p.xs_off + i * 16);
                h.x = cvt_bf16x2_f16x2(v.x);
                h.y = cvt_bf16x2_f16x2(v.y);
                h.z = cvt_bf16x2_f16x2(v.z);
                h.w = cvt_bf16x2_f16x2(v.w);
            }
            *reinterpret_cast<uint4*>(smem + p.xs_off + i * 16) = h;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
    }

    const int g = lane >> 2, tq = lane & 3;
    const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
    const int tile = warp % kTiles, my_half = warp / kTiles;
    const int r_lo = 16 * tile + 2 * g, r_hi = r_lo + 1;
    uint32_t off_lo[4], off_hi[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int chunk = 2 * j + (tq >> 1);
        off_lo[j] = r_lo * 128 + ((chunk ^ (r_lo & 7)) << 4) + (tq & 1) * 8;
        off_hi[j] = r_hi * 128 + ((chunk ^ (r_hi & 7)) << 4) + (tq & 1) * 8;
    }

    float acc_lo = 0.f, acc_hi = 0.f;
    uint4 xa[4], xb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) xa[j] = xb[j] = make_uint4(0u, 0u, 0u, 0u);
    long long u = u0;
    int strip = static_cast<int>(u / p.KS), ks = static_cast<int>(u % p.KS);
    int cur = strip;
    float* pair_buf = reinterpret_cast<float*>(smem + p.pair_off) + tile * 32;
    auto flush = [&](int st) {
        if (kHalves == 2) {
            // the second half hands its partial sums to the first
            if (my_half == 1 && tq == 0) {
                pair_buf[2 * g] = acc_lo;
                pair_buf[2 * g + 1] = acc_hi;
            }
            asm volatile("bar.sync %0, 64;" ::"r"(2 + tile) : "memory");
            if (my_half == 1) {
                asm volatile("bar.sync %0, 64;" ::"r"(2 + tile) : "memory");
                return;
            }
            if (tq == 0) {
                acc_lo += pair_buf[2 * g];
                acc_hi += pair_buf[2 * g + 1];
            }
            asm volatile("bar.sync %0, 64;" ::"r"(2 + tile) : "memory");
        }
        if (tq != 0) return;
        const bool whole = static_cast<long long>(st) * p.KS >= u0 &&
                           static_cast<long long>(st + 1) * p.KS <= u1;
        const int n_lo = st * kR + r_lo, n_hi = n_lo + 1;
        if (whole) {
            if (n_lo < p.N) p.y[n_lo] = acc_lo;
            if (n_hi < p.N) p.y[n_hi] = acc_hi;
        } else {
            if (n_lo < p.N) red_add_f32(p.y + n_lo, acc_lo);
            if (n_hi < p.N) red_add_f32(p.y + n_hi, acc_hi);
        }
    };

    int slot = 0;
    uint32_t fparity = 0;
    for (; u < u1; ++u) {
        if (strip != cur) {
            flush(cur);
            acc_lo = acc_hi = 0.f;
            cur = strip;
        }
        if (!mbar_wait(full(slot), fparity)) {
            if (lane == 0) atomicOr(&g_gemv_tma_error, 2u);
            return;
        }
        // Groups past K have zero codes (TMA fill), zero scales and zero x,
        // and add exactly 0.
        const uint32_t coff = kLutBytes + slot * kCodeStageBytes;
        const uint32_t soff = p.scale_off + slot * kScaleStageBytes;
        const uint4 sl = ld_smem<uint4>(smem, soff + r_lo * 16);
        const uint4 sh = ld_smem<uint4>(smem, soff + r_hi * 16);
#pragma unroll
        for (int hh = 0; hh < 2 / kHalves; ++hh) {
            const int half = (kHalves == 2) ? my_half : hh;
            // scale words of this half: groups 4 half .. 4 half + 3
            const uint32_t sl0 = half ? sl.z : sl.x, sl1 = half ? sl.w : sl.y;
            const uint32_t sh0 = half ? sh.z : sh.x, sh1 = half ? sh.w : sh.y;
            uint2 clo[4], chi[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                clo[j] = ld_smem<uint2>(smem, coff + half * kBoxBytes + off_lo[j]);
                chi[j] = ld_smem<uint2>(smem, coff + half * kBoxBytes + off_hi[j]);
                // Only column 0 of the B operand (lanes 0-3) is read back; the
                // other lanes keep stale x, which only feeds unused columns.
                if (g == 0) {
                    const uint32_t xo = p.xs_off + (ks * kSG + 4 * half + j) * 128 + tq * 32;
                    xa[j] = ld_smem<uint4>(smem, xo);
                    xb[j] = ld_smem<uint4>(smem, xo + 16);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float d0, d2;
                group_mma(smem, clo[j], chi[j], xa[j], xb[j], lane4, d0, d2);
                const uint32_t wl = (j < 2) ? sl0 : sl1, wh = (j < 2) ? sh0 : sh1;
                const float s_lo = (j & 1) ? half_hi(wl) : half_lo(wl);
                const float s_hi = (j & 1) ? half_hi(wh) : half_lo(wh);
                acc_lo = fmaf(s_lo, d0, acc_lo);
                acc_hi = fmaf(s_hi, d2, acc_hi);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(slot));
        if (++slot == S) {
            slot = 0;
            fparity ^= 1u;
        }
        if (++ks == p.KS) {
            ks = 0;
            ++strip;
        }
    }
    flush(cur);
}

}  // namespace

// Returns cudaErrorNotSupported when the shape does not fit this kernel (the
// caller then uses the general small-M kernel).
cudaError_t take_gemv_tma_error(unsigned int* out) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_gemv_tma_error, sizeof(unsigned int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_gemv_tma_error, &zero, sizeof(unsigned int));
    return e;
}

cudaError_t launch_gemv_tma(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                            const uint16_t* x, float* y, int64_t N, int64_t K, cudaStream_t s,
                            const DeviceInfo& dev) {
    TmaGemv p{};
    p.scales = scales;
    p.cb = cb;
    p.x = x;
    p.y = y;
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.G = static_cast<int>(K / kGroup);
    p.KS = (p.G + kSG - 1) / kSG;
    p.strips = static_cast<int>((N + kR - 1) / kR);
    const int x_bytes = p.KS * kSG * kGroup * 2;
    const int per_stage = kCodeStageBytes + kScaleStageBytes;
    const int fixed = kLutBytes + x_bytes + 32 + kTiles * 128 + (2 * kMaxStages + 1) * 8 + 1024;
    int S = (dev.smem_optin - fixed) / per_stage;
    if (S > kMaxStages) S = kMaxStages;
    if (S < 2) return cudaErrorNotSupported;
    p.stages = S;
    p.scale_off = kLutBytes + S * kCodeStageBytes;
    p.xs_off = p.scale_off + S * kScaleStageBytes;
    p.cb_off = p.xs_off + x_bytes;
    p.pair_off = p.cb_off + 32;
    p.bar_off = p.pair_off + kTiles * 32 * 4;
    const int smem = p.bar_off + (2 * S + 1) * 8;

    const int mode = (p.G % 8 == 0) ? kScaleTma : (p.G % 4 == 0) ? kScaleAsync : kScaleSync;
    CUtensorMap cmap, smap;
    cudaError_t e = encode_tensor_map_2d(&cmap, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                                         static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2),
                                         static_cast<uint64_t>(K / 2), kR, 128,
                                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    if (mode == kScaleTma) {
        e = encode_tensor_map_2d(&smap, scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                                 static_cast<uint64_t>(N), static_cast<uint64_t>(p.G),
                                 static_cast<uint64_t>(p.G) * 2, kR, kSG,
                                 CU_TENSOR_MAP_SWIZZLE_NONE);
        if (e != cudaSuccess) return e;
    } else {
        smap = cmap;  // unused
    }

    const long long U = static_cast<long long>(p.strips) * p.KS;
    const int grid = static_cast<int>(U < dev.sm_count ? U : dev.sm_count);
    bool split = false;
    for (int c = 1; c < grid && !split; ++c)
        if ((U * c / grid) % p.KS != 0) split = true;
    if (split) {
        e = cudaMemsetAsync(y, 0, static_cast<size_t>(N) * sizeof(float), s);
        if (e != cudaSuccess) return e;
    }
    const void* fn = mode == kScaleTma     ? reinterpret_cast<const void*>(gemv_tma_kernel<kScaleTma>)
                     : mode == kScaleAsync ? reinterpret_cast<const void*>(gemv_tma_kernel<kScaleAsync>)
                                           : reinterpret_cast<const void*>(gemv_tma_kernel<kScaleSync>);
    e = ensure_smem_attr(fn, smem, 8 + mode, dev.device);
    if (e != cudaSuccess) return e;
    if (mode == kScaleTma)
        gemv_tma_kernel<kScaleTma><<<grid, kThreads, smem, s>>>(cmap, smap, p);
    else if (mode == kScaleAsync)
        gemv_tma_kernel<kScaleAsync><<<grid, kThreads, smem, s>>>(cmap, smap, p);
    else
        gemv_tma_kernel<kScaleSync><<<grid, kThreads, smem, s>>>(cmap, smap, p);
    return cudaGetLastError();
}

}  // namespace q4
