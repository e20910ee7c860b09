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
#include "q4_sm100.cuh"

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
        if (!Q4_IN_BOUNDS(n * K + g * kGroup, kGroup, N * K) ||
            !Q4_IN_BOUNDS(n * (K / 4) + g * (kGroup / 4), kGroup / 4, N * (K / 4)) ||
            !Q4_IN_BOUNDS(n * G + g, 1, N * G))
            continue;
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
        if (!Q4_IN_BOUNDS(n * (K / 4) + j * 4, 4, N * (K / 4)) || !Q4_IN_BOUNDS(n * G + k0 / kGroup, 1, N * G) ||
            !Q4_IN_BOUNDS(n * K + k0, 16, N * K))
            continue;
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
            if (ra < N && Q4_IN_BOUNDS(ra * (K / 4) + grp * 16, 16, N * (K / 4)) &&
                Q4_IN_BOUNDS(ra * G + grp, 1, N * G)) {
                c.wa = __ldcs(reinterpret_cast<const uint4*>(codes + ra * (K / 4) + grp * 16));
                c.sa = __ldg(reinterpret_cast<const unsigned short*>(scales + ra * G + grp));
            }
            if (rb < N && Q4_IN_BOUNDS(rb * (K / 4) + grp * 16, 16, N * (K / 4)) &&
                Q4_IN_BOUNDS(rb * G + grp, 1, N * G)) {
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
        const __half h = __float2half_rn(bf16_bits_to_float(Q4_IN_BOUNDS(k, 1, K) ? __ldg(x + k) : 0));
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
            if (ra < N && Q4_IN_BOUNDS(ra, 1, N)) atomicAdd(y + ra, va);
            if (rb < N && Q4_IN_BOUNDS(rb, 1, N)) atomicAdd(y + rb, vb);
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

// ---------------------------------------------------------------------------
// gemv2 on a bulk-copy ring (the path for K <= kR2MaxK)
// ---------------------------------------------------------------------------
// Weight stream: CTA c owns the rows [N c / grid, N (c + 1) / grid); a
// producer warp copies 16-row tiles of their codes into a shared-memory ring
// with 1-D bulk copies (one contiguous copy per tile when a row is at most
// 2 KB, else one ~2 KB segment per row per stage), and the stage's scales
// with cp.async beside them; both complete on the stage's mbarrier.
//
// Consumer warp w takes unit w of every stage: 16 rows x 128 code bytes
// (8 groups, 512 k).  Lane (g, tq) reads 32 bytes of rows g and g + 8: group
// 2 tq ("lo") and group 2 tq + 1 ("hi") of the unit.  MMA (q, i, h), 32 per
// unit, takes from word q of each of those four 16-byte groups the codes at
// bit position 2 i of bytes 2 h and 2 h + 1, i.e. k = 16 q + 8 h + 4 e + i
// (e = 0, 1) of the group, rebuilt by one PRMT each from the codebook held as
// split low and high bytes; the selector of four codes is
// (word & (3 << 2 i) per byte) * 0x11 >> 2 i + 0x40 per byte (one LOP and
// one IMAD).  a0 / a2 carry row g's lo / hi group, a1 / a3 row g + 8's.
//
// Groups as B columns: B column n holds x of the unit's group n and zeros
// elsewhere, so the accumulator column n is group n's partial sum and lane
// (g, tq) holds exactly its own two groups (columns 2 tq, 2 tq + 1) of rows g
// and g + 8, which it scales in fp32 with those groups' scales.  In the B
// fragment only lane (2 tq, tq) has a nonzero b0 and lane (2 tq + 1, tq) a
// nonzero b1: every lane holds the binary16 x of group g of its unit and
// multiplies it by a per-lane 1.0 / 0.0 half2 mask (HMUL2, on the FMA pipe)
// into b0 and b1.  Products are exact and sums fp32, as in q4_gemv.
//
// A warp keeps its units' sums of a tile in its own shared-memory slot; at
// the end of a pass of tiles the CTA adds the slots and writes each y element
// once (no memset, no atomics).  Programmatic dependent launch as q4_gemv.
constexpr int kR2CW = 16;                      // consumer warps
constexpr int kR2Threads = (kR2CW + 1) * 32;   // + one producer warp
constexpr int kR2Unit = 128;                   // code bytes of a row per unit
constexpr int kR2MaxKC = 2048;                 // code bytes of a row per stage
constexpr int kR2MaxStages = 6;
constexpr int kR2MinPassTiles = 4;
constexpr int kR2MaxPassTiles = 64;
constexpr uint32_t kR2TileSlotBytes = kR2CW * 16 * 4;

__device__ unsigned int g_gemv2_error;

// The multiplier of the selector arithmetic (0x11) is passed as a kernel
// argument so that it stays one integer multiply-add (the FMA pipe) instead of
// being folded into a shift and an add (the ALU pipe, which the PRMTs keep
// busy).
struct SelMul {
    uint32_t k11;  // 0x11: a code c in bits 0-1 of a byte becomes c | c << 4
};

struct G2 {
    const uint8_t* codes;
    const uint16_t* scales;
    const uint16_t* cb;
    const uint16_t* x;
    float* y;
    int N, K, G;
    int R;      // code bytes of a row (K / 4)
    int KC;     // code bytes of a row per stage (the ring's row pitch)
    int GS;     // groups of a row per stage (KC / 16)
    int C;      // stages per 16-row tile
    int NS;     // ring stages
    int PT;     // tiles per pass of the partial slots
    int units;  // units of a row (ceil(R / 128))
    uint32_t slot_off;  // per-warp row partials (after the table when there is one)
    uint32_t bar_off, x_off, zero_off, ring_off, stage_bytes, scale_off;
    SelMul k;
};

// Dynamic shared memory starts at this shared-window address on sm_100 (the
// launcher checks the device's reservation), so a table at its start is read
// with the address in the load's immediate.
constexpr uint32_t kR2Base = 1024;
constexpr uint32_t kR2LutBytes = 65536;  // 256 byte values x 32 lanes x 8 bytes

// Table entry of code byte `byte` of w for this lane: the binary16 pairs
// (cb[c0], cb[c1]) and (cb[c2], cb[c3]) of its four codes.
template <int kByte>
__device__ __forceinline__ uint2 lut2(uint32_t w, uint32_t lane8) {
    uint2 v;
    asm("ld.shared.v2.b32 {%0, %1}, [%2 + %3];"
        : "=r"(v.x), "=r"(v.y)
        : "r"(__byte_perm(w, lane8, 0x5504 | (kByte << 4))), "n"(kR2Base));
    return v;
}

__device__ __forceinline__ uint4 lds128_v(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t word4(const uint4& v, int q) {
    return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}

__device__ __forceinline__ uint32_t madlo(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// PRMT selectors for the four codes at bit position 2 i of the bytes of w:
// the low 16 bits of *s0 pick bytes 0 and 1, those of *s1 bytes 2 and 3, as
// (cb[c] low byte, cb[c] high byte) pairs.  PRMT nibble c picks the
// codebook's low byte of entry c and 4 + c its high byte, so a code c becomes
// the selector byte c * 0x11 + 0x40; each code is moved to bits 0-1 of its
// byte first, so no product carries into the next byte.  (Measured on B200:
// folding the shift into the high half of a product, mad.hi, cost about a
// quarter more time, as it is not one instruction.)
template <int kI>
__device__ __forceinline__ void selectors(uint32_t w, const SelMul& k, uint32_t* s0, uint32_t* s1) {
    const uint32_t t = (w >> (2 * kI)) & 0x03030303u;
    *s0 = madlo(t, k.k11, 0x40404040u);
    *s1 = *s0 >> 16;
}

// binary16 pair (lo, hi) from two bfloat16 values
__device__ __forceinline__ uint32_t bf16pair_to_f16x2(uint32_t lo, uint32_t hi) {
    const __half2 h = __floats2half2_rn(__uint_as_float(lo << 16), __uint_as_float(hi << 16));
    return *reinterpret_cast<const uint32_t*>(&h);
}

template <int kSW>
__device__ __forceinline__ void copy_scales(uint32_t dst, const uint16_t* src) {
    if (kSW == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
    else if (kSW == 8)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
    else if (kSW == 4)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
    else
        sts_u16(dst, __ldg(reinterpret_cast<const unsigned short*>(src)));
}

// kWhole: a tile is one stage (rows of at most 2 KB); kSW: bytes per scale
// copy (16, 8, 4 with cp.async; 2 = plain loads, for an odd group count).
// kLut: the word quarters q < kR2LutQuarters of every group are decoded
// through a per-lane byte -> four binary16 values table in shared memory (one
// LDS.64 and one PRMT per four weights) instead of by PRMT from the codebook
// registers (about 2.4 ALU instructions per weight), which moves the decode
// from the ALU pipe to the shared-memory pipe.  Measured on B200 (70B
// linears): table for 2 quarters 63.9 us on gate_up, 3: 62.3, 4: 61.4.
constexpr int kR2LutQuarters = 4;  // quarters decoded through the table when kLut

template <bool kWhole, int kSW, bool kLut>
__global__ void __launch_bounds__(kR2Threads, 1) gemv2_ring_kernel(const G2 p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tq = lane & 3;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const uint32_t base = smem_u32(smem);
    if (kLut && base != kR2Base) {
        // the table's immediate addressing does not hold: report, write nothing
        if (tid == 0) atomicOr(&g_gemv2_error, 0x1u);
        return;
    }
    const uint32_t bars = base + p.bar_off;
    const int NS = p.NS;
    const int r0 = static_cast<int>(static_cast<int64_t>(p.N) * blockIdx.x / gridDim.x);
    const int r1 = static_cast<int>(static_cast<int64_t>(p.N) * (blockIdx.x + 1) / gridDim.x);
    const int nrows = r1 - r0;
    const int T = (nrows + 15) >> 4;
    const int total = T * p.C;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bars + 8u * s, 33);             // expect_tx + the producer lanes' scale copies
            mbar_init(bars + 8u * (NS + s), kR2CW);   // one arrival per consumer warp
        }
        fence_mbar_init();
    }
    // warm L2 with the first tile, its scales and x while the preceding kernel finishes
    if (warp == kR2CW && total > 0) {
        const int rows = min(16, nrows);
        if (kWhole) {
            if (lane == 0)
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.codes + static_cast<int64_t>(r0) * p.R),
                             "r"(static_cast<uint32_t>(rows * p.R)) : "memory");
        } else if (lane < rows) {
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.codes + static_cast<int64_t>(r0 + lane) * p.R),
                         "r"(static_cast<uint32_t>(min(p.KC, p.R))) : "memory");
        }
        if (lane == 31)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.x), "r"(static_cast<uint32_t>(p.K) * 2u)
                         : "memory");
    }
    __syncthreads();

    if (warp == kR2CW) {
        // ------------------------------ producer ------------------------------
        asm volatile("griddepcontrol.wait;" ::: "memory");
        int slot = 0, t = 0, c = 0;
        uint32_t eparity = 1;
        int issued = 0;
        for (int i = 0; i < total; ++i) {
            if (i >= NS) {
                uint32_t ok = 1;
                if (lane == 0) ok = mbar_wait(bars + 8u * (NS + slot), eparity) ? 1u : 0u;
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) {
                    if (lane == 0) atomicOr(&g_gemv2_error, 0x2u);
                    break;
                }
            }
            const int rows = min(16, nrows - 16 * t);
            const int row0 = r0 + 16 * t;
            const uint32_t dst = base + p.ring_off + slot * p.stage_bytes;
            const uint32_t full = bars + 8u * slot;
            const int cbytes = kWhole ? p.R : min(p.KC, p.R - c * p.KC);
            if (lane == 0) mbar_arrive_expect_tx(full, static_cast<uint32_t>(rows * cbytes));
            __syncwarp();
            [[maybe_unused]] const int64_t code_extent = static_cast<int64_t>(p.N) * p.R;
            if (kWhole) {
                if (lane == 0 && Q4_IN_BOUNDS(static_cast<int64_t>(row0) * p.R, rows * p.R, code_extent))
                    bulk_load(dst, p.codes + static_cast<int64_t>(row0) * p.R, static_cast<uint32_t>(rows * p.R), full);
            } else if (lane < rows &&
                       Q4_IN_BOUNDS(static_cast<int64_t>(row0 + lane) * p.R + c * p.KC, cbytes, code_extent)) {
                bulk_load(dst + lane * p.KC, p.codes + static_cast<int64_t>(row0 + lane) * p.R + c * p.KC,
                          static_cast<uint32_t>(cbytes), full);
            }
            // scales of the stage: rows x ng groups, row pitch GS in the stage
            const int g0 = kWhole ? 0 : c * p.GS;
            const int ng = kWhole ? p.G : min(p.GS, p.G - g0);
            const int per_row = ng * 2 / kSW;
            const uint32_t sdst = dst + p.scale_off;
            for (int j = lane; j < rows * per_row; j += 32) {
                const int r = j / per_row, q = j - r * per_row;
                if (Q4_IN_BOUNDS(static_cast<int64_t>(row0 + r) * p.G + g0 + q * (kSW / 2), kSW / 2,
                                 static_cast<int64_t>(p.N) * p.G))
                    copy_scales<kSW>(sdst + r * (p.GS * 2) + q * kSW,
                                 p.scales + static_cast<int64_t>(row0 + r) * p.G + g0 + q * (kSW / 2));
            }
            if (kSW > 2)
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(full) : "memory");
            else
                mbar_arrive(full);
            ++issued;
            if (++c == p.C) {
                c = 0;
                ++t;
            }
            if (++slot == NS) {
                slot = 0;
                eparity ^= 1u;
            }
        }
        // leave only once this warp's copies have landed (bounded)
        if (lane == 0) {
            for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i)
                if (!mbar_wait(bars + 8u * (i % NS), (i / NS) & 1)) {
                    atomicOr(&g_gemv2_error, 0x4u);
                    break;
                }
        }
        return;
    }

    // ------------------------------- consumers ------------------------------
    float* acc_s = reinterpret_cast<float*>(smem + p.slot_off);  // [PT tiles][kR2CW warps][16 rows]
    const int upk = kWhole ? p.units : p.KC / kR2Unit;
    const uint32_t off1 = 32 * tq + 16 * (g & 1), off2 = 32 * tq + 16 * (1 - (g & 1));
    const bool swap = (g & 1) != 0;
    const uint32_t rowA = static_cast<uint32_t>(g * p.KC), rowB = static_cast<uint32_t>((g + 8) * p.KC);
    // B operand: b0 carries x for lane (2 tq, tq) and b1 for lane (2 tq + 1,
    // tq); every other b register reads the zero block
    const bool act0 = g == 2 * tq, act1 = g == 2 * tq + 1;
    const SelMul km = p.k;

    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint32_t cbl = 0, cbh = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t hv = __ldg(p.cb + e);
        cbl |= (hv & 0xFFu) << (8 * e);
        cbh |= (hv >> 8) << (8 * e);
    }
    {
        // x of every unit as binary16 in MMA order, at x_off + 1024 u +
        // 128 (m / 4) + 16 a + 4 (m % 4) for MMA m = 8 q + 2 i + h of group
        // 8 u + a; zeros past the last group.  A quarter decoded by PRMT
        // takes code i of bytes 2 h, 2 h + 1 of its word: (x[16 q + 8 h + i],
        // x[16 q + 8 h + 4 + i]).  A quarter decoded by the table takes codes
        // 2 h, 2 h + 1 of byte i: (x[16 q + 4 i + 2 h], x[16 q + 4 i + 2 h + 1]).
        const int items = p.units * 8 * 4;  // (unit, a, q)
        for (int it = tid; it < items; it += kR2CW * 32) {
            const int q = it & 3, a = (it >> 2) & 7, u = it >> 5;
            const int grp = 8 * u + a;
            uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
            if (grp < p.G && Q4_IN_BOUNDS(static_cast<int64_t>(grp) * kGroup + 16 * q, 16, p.K)) {
                const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(grp) * kGroup + 16 * q);
                v0 = __ldg(src);
                v1 = __ldg(src + 1);
            }
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            const bool by_table = kLut && q < kR2LutQuarters;
#pragma unroll
            for (int mm = 0; mm < 8; ++mm) {
                const int i = mm >> 1, h = mm & 1, m = 8 * q + mm;
                uint32_t pair;
                if (by_table) {
                    pair = bf16pair_to_f16x2(w[2 * i + h] & 0xFFFFu, w[2 * i + h] >> 16);
                } else {
                    const int e0 = 8 * h + i, e1 = 8 * h + 4 + i;
                    pair = bf16pair_to_f16x2((w[e0 >> 1] >> (16 * (e0 & 1))) & 0xFFFFu,
                                             (w[e1 >> 1] >> (16 * (e1 & 1))) & 0xFFFFu);
                }
                *reinterpret_cast<uint32_t*>(smem + p.x_off + 1024 * u + 128 * (m >> 2) + 16 * a + 4 * (m & 3)) = pair;
            }
        }
        if (kLut) {
            // entry of byte value v for lane l at 256 v + 8 l: (cb[c0], cb[c1]), (cb[c2], cb[c3])
            for (int it = tid; it < 256 * 16; it += kR2CW * 32) {
                const int v = it >> 4;
                const uint32_t c0 = __ldg(p.cb + (v & 3)), c1 = __ldg(p.cb + ((v >> 2) & 3));
                const uint32_t c2 = __ldg(p.cb + ((v >> 4) & 3)), c3 = __ldg(p.cb + (v >> 6));
                const uint32_t e01 = c0 | (c1 << 16), e23 = c2 | (c3 << 16);
                *reinterpret_cast<uint4*>(smem + 256 * v + 16 * (it & 15)) = make_uint4(e01, e23, e01, e23);
            }
        }
        for (int it = tid; it < 1024 / 16; it += kR2CW * 32)
            *reinterpret_cast<uint4*>(smem + p.zero_off + 16 * it) = make_uint4(0u, 0u, 0u, 0u);
        asm volatile("bar.sync 1, %0;" ::"n"(kR2CW * 32) : "memory");
    }

    bool bad = false;
    int slot = 0;
    uint32_t fparity = 0;
    for (int pt0 = 0; pt0 < T; pt0 += p.PT) {
        const int pt1 = min(T, pt0 + p.PT);
        for (int t = pt0; t < pt1; ++t) {
            float acc_g = 0.f, acc_h = 0.f;  // rows g and g + 8
            for (int c = 0; c < p.C; ++c) {
                if (!bad && !mbar_wait(bars + 8u * slot, fparity)) {
                    bad = true;
                    if (lane == 0) atomicOr(&g_gemv2_error, 0x8u);
                }
                const int U = c * upk + warp;  // unit of the row
                if (!bad && warp < upk && U < p.units) {
                    const uint32_t sb = base + p.ring_off + slot * p.stage_bytes;
                    // x of group 8 U + g for the active lanes, the zero block for the rest
                    const uint32_t xg = base + p.x_off + 1024 * U + 16 * g, xz = base + p.zero_off;
                    const uint32_t xa0 = act0 ? xg : xz, xa1 = act1 ? xg : xz;
                    const uint32_t ua = sb + warp * kR2Unit;
                    const uint4 a1 = lds128_v(ua + rowA + off1), a2 = lds128_v(ua + rowA + off2);
                    const uint4 b1 = lds128_v(ua + rowB + off1), b2 = lds128_v(ua + rowB + off2);
                    const uint4 lo_g = swap ? a2 : a1, hi_g = swap ? a1 : a2;
                    const uint4 lo_h = swap ? b2 : b1, hi_h = swap ? b1 : b2;
                    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 xv0 = lds128_v(xa0 + 256 * q), xv1 = lds128_v(xa0 + 256 * q + 128);
                        const uint4 xw0 = lds128_v(xa1 + 256 * q), xw1 = lds128_v(xa1 + 256 * q + 128);
                        const uint32_t xb0[8] = {xv0.x, xv0.y, xv0.z, xv0.w, xv1.x, xv1.y, xv1.z, xv1.w};
                        const uint32_t xb1[8] = {xw0.x, xw0.y, xw0.z, xw0.w, xw1.x, xw1.y, xw1.z, xw1.w};
                        const uint32_t wlg = word4(lo_g, q), whg = word4(hi_g, q);
                        const uint32_t wlh = word4(lo_h, q), whh = word4(hi_h, q);
                        if (kLut && q < kR2LutQuarters) {
                            const uint32_t lane8 = static_cast<uint32_t>(lane) * 8u;
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                uint2 tlg, tlh, thg, thh;
                                switch (i) {
                                    case 0:
                                        tlg = lut2<0>(wlg, lane8); tlh = lut2<0>(wlh, lane8);
                                        thg = lut2<0>(whg, lane8); thh = lut2<0>(whh, lane8);
                                        break;
                                    case 1:
                                        tlg = lut2<1>(wlg, lane8); tlh = lut2<1>(wlh, lane8);
                                        thg = lut2<1>(whg, lane8); thh = lut2<1>(whh, lane8);
                                        break;
                                    case 2:
                                        tlg = lut2<2>(wlg, lane8); tlh = lut2<2>(wlh, lane8);
                                        thg = lut2<2>(whg, lane8); thh = lut2<2>(whh, lane8);
                                        break;
                                    default:
                                        tlg = lut2<3>(wlg, lane8); tlh = lut2<3>(wlh, lane8);
                                        thg = lut2<3>(whg, lane8); thh = lut2<3>(whh, lane8);
                                        break;
                                }
                                uint32_t a[4] = {tlg.x, tlh.x, thg.x, thh.x};
                                mma_16816(d0, a, xb0[2 * i], xb1[2 * i], d0);
                                uint32_t a2[4] = {tlg.y, tlh.y, thg.y, thh.y};
                                mma_16816(d1, a2, xb0[2 * i + 1], xb1[2 * i + 1], d1);
                            }
                            continue;
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint32_t slg0, slg1, shg0, shg1, slh0, slh1, shh0, shh1;
                            switch (i) {
                                case 0:
                                    selectors<0>(wlg, km, &slg0, &slg1); selectors<0>(whg, km, &shg0, &shg1);
                                    selectors<0>(wlh, km, &slh0, &slh1); selectors<0>(whh, km, &shh0, &shh1);
                                    break;
                                case 1:
                                    selectors<1>(wlg, km, &slg0, &slg1); selectors<1>(whg, km, &shg0, &shg1);
                                    selectors<1>(wlh, km, &slh0, &slh1); selectors<1>(whh, km, &shh0, &shh1);
                                    break;
                                case 2:
                                    selectors<2>(wlg, km, &slg0, &slg1); selectors<2>(whg, km, &shg0, &shg1);
                                    selectors<2>(wlh, km, &slh0, &slh1); selectors<2>(whh, km, &shh0, &shh1);
                                    break;
                                default:
                                    selectors<3>(wlg, km, &slg0, &slg1); selectors<3>(whg, km, &shg0, &shg1);
                                    selectors<3>(wlh, km, &slh0, &slh1); selectors<3>(whh, km, &shh0, &shh1);
                                    break;
                            }
                            uint32_t a[4];
                            a[0] = __byte_perm(cbl, cbh, slg0);
                            a[1] = __byte_perm(cbl, cbh, slh0);
                            a[2] = __byte_perm(cbl, cbh, shg0);
                            a[3] = __byte_perm(cbl, cbh, shh0);
                            mma_16816(d0, a, xb0[2 * i], xb1[2 * i], d0);
                            a[0] = __byte_perm(cbl, cbh, slg1);
                            a[1] = __byte_perm(cbl, cbh, slh1);
                            a[2] = __byte_perm(cbl, cbh, shg1);
                            a[3] = __byte_perm(cbl, cbh, shh1);
                            mma_16816(d1, a, xb0[2 * i + 1], xb1[2 * i + 1], d1);
                        }
                    }
                    // columns 2 tq, 2 tq + 1: this lane's groups of rows g, g + 8
                    const int gl = warp * 8 + 2 * tq;  // group index within the stage's scale rows
                    const int ga = U * 8 + 2 * tq;      // group index within the row
                    const uint32_t srow_g = sb + p.scale_off + g * (p.GS * 2) + 2 * gl;
                    const uint32_t srow_h = srow_g + 8 * (p.GS * 2);
                    float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;
                    if (ga < p.G) {
                        s00 = __half2float(__ushort_as_half(ld_smem<uint16_t>(smem, srow_g - base)));
                        s10 = __half2float(__ushort_as_half(ld_smem<uint16_t>(smem, srow_h - base)));
                    }
                    if (ga + 1 < p.G) {
                        s01 = __half2float(__ushort_as_half(ld_smem<uint16_t>(smem, srow_g - base + 2)));
                        s11 = __half2float(__ushort_as_half(ld_smem<uint16_t>(smem, srow_h - base + 2)));
                    }
                    acc_g = fmaf(s00, d0[0] + d1[0], acc_g);
                    acc_g = fmaf(s01, d0[1] + d1[1], acc_g);
                    acc_h = fmaf(s10, d0[2] + d1[2], acc_h);
                    acc_h = fmaf(s11, d0[3] + d1[3], acc_h);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + 8u * (NS + slot));
                if (++slot == NS) {
                    slot = 0;
                    fparity ^= 1u;
                }
            }
            // the four lanes of a row hold its eight groups' sums
            acc_g += __shfl_xor_sync(0xFFFFFFFFu, acc_g, 1);
            acc_g += __shfl_xor_sync(0xFFFFFFFFu, acc_g, 2);
            acc_h += __shfl_xor_sync(0xFFFFFFFFu, acc_h, 1);
            acc_h += __shfl_xor_sync(0xFFFFFFFFu, acc_h, 2);
            if (tq == 0) {
                float* slot_w = acc_s + ((t - pt0) * kR2CW + warp) * 16;
                slot_w[g] = acc_g;
                slot_w[g + 8] = acc_h;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kR2CW * 32) : "memory");
        const int row_end = min(nrows, 16 * pt1);
        for (int r = 16 * pt0 + tid; r < row_end; r += kR2CW * 32) {
            const int rl = r - 16 * pt0;
            const float* q = acc_s + (rl >> 4) * kR2CW * 16 + (rl & 15);
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < kR2CW; ++w) sum += q[16 * w];
            if (Q4_IN_BOUNDS(r0 + r, 1, p.N)) p.y[r0 + r] = sum;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kR2CW * 32) : "memory");
    }
}

template <bool kWhole, int kSW, bool kLut>
cudaError_t launch_ring2(const G2& p, int grid, int smem, int slot, cudaStream_t s, const DeviceInfo& dev) {
    auto kern = gemv2_ring_kernel<kWhole, kSW, kLut>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem, slot, dev.device);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kR2Threads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

// Plans and launches the ring kernel; cudaErrorNotSupported when the shape
// does not fit its shared-memory layout (x of a long row plus the ring).
cudaError_t launch_gemv2_ring(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                              const uint16_t* x, float* y, int64_t N, int64_t K, cudaStream_t s,
                              const DeviceInfo& dev) {
    G2 p{};
    p.codes = codes;
    p.scales = scales;
    p.cb = cb;
    p.x = x;
    p.y = y;
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.G = static_cast<int>(K / kGroup);
    p.R = static_cast<int>(K / 4);
    p.k = SelMul{0x11u};
    p.units = (p.R + kR2Unit - 1) / kR2Unit;
    const bool whole = p.R <= kR2MaxKC;
    if (whole) {
        p.C = 1;
        p.KC = p.R;
        p.GS = p.G;
    } else {
        p.C = (p.R + kR2MaxKC - 1) / kR2MaxKC;
        p.KC = ((p.R + p.C - 1) / p.C + kR2Unit - 1) / kR2Unit * kR2Unit;
        p.C = (p.R + p.KC - 1) / p.KC;
        p.GS = p.KC / 16;
    }
    const uint32_t code_bytes = (static_cast<uint32_t>(16 * p.KC) + 127u) & ~127u;
    p.scale_off = code_bytes;
    p.stage_bytes = code_bytes + ((static_cast<uint32_t>(16 * p.GS * 2) + 127u) & ~127u);
    const uint32_t x_bytes = static_cast<uint32_t>(p.units) * 1024u;
    uint32_t head = 0;  // the table, when there is one, ahead of everything else
    auto layout = [&](int pt) {
        p.PT = pt;
        p.slot_off = head;
        p.bar_off = head + static_cast<uint32_t>(pt) * kR2TileSlotBytes;
        p.zero_off = p.bar_off + 128u;
        p.x_off = p.zero_off + 1024u;
        p.ring_off = (p.x_off + x_bytes + 127u) & ~127u;
        return dev.smem_optin - static_cast<int>(p.ring_off);
    };
    // the table needs the dynamic shared-memory base at kR2Base and room for
    // at least three ring stages beside it
    bool lut = dev.smem_reserved == static_cast<int>(kR2Base);
    if (lut) {
        head = kR2LutBytes;
        lut = layout(kR2MinPassTiles) / static_cast<int>(p.stage_bytes) >= 3;
    }
    if (!lut) head = 0;
    int ns = layout(kR2MinPassTiles) / static_cast<int>(p.stage_bytes);
    if (ns > kR2MaxStages) ns = kR2MaxStages;
    if (ns < 2) return cudaErrorNotSupported;
    p.NS = ns;
    const int64_t tiles_per_cta = ((N + dev.sm_count - 1) / dev.sm_count + 15) / 16 + 1;
    const int pt_cap = static_cast<int>(tiles_per_cta < kR2MaxPassTiles ? tiles_per_cta : kR2MaxPassTiles);
    int pt = pt_cap < kR2MinPassTiles ? kR2MinPassTiles : pt_cap;
    while (pt > kR2MinPassTiles && layout(pt) < ns * static_cast<int>(p.stage_bytes)) --pt;
    layout(pt);
    const int smem = static_cast<int>(p.ring_off + ns * p.stage_bytes);
    if (smem > dev.smem_optin) return cudaErrorNotSupported;
    const int64_t tiles = (N + 15) / 16;
    const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
    // widest scale copy that every source and destination offset allows
    const int gcd_groups = p.G % 8 == 0 && p.GS % 8 == 0 ? 8 : (p.G % 4 == 0 && p.GS % 4 == 0 ? 4 : (p.G % 2 == 0 && p.GS % 2 == 0 ? 2 : 1));
    // slots 51..58 without the table, 59..66 with it
    const int slot = 51 + (whole ? 0 : 4) + (gcd_groups == 8 ? 0 : gcd_groups == 4 ? 1 : gcd_groups == 2 ? 2 : 3) +
                     (lut ? 8 : 0);
#define Q4_RING2(W, SW)                                                                  \
    return lut ? launch_ring2<W, SW, true>(p, grid, smem, slot, s, dev)                  \
               : launch_ring2<W, SW, false>(p, grid, smem, slot, s, dev)
    if (whole) {
        switch (gcd_groups) {
            case 8: Q4_RING2(true, 16);
            case 4: Q4_RING2(true, 8);
            case 2: Q4_RING2(true, 4);
            default: Q4_RING2(true, 2);
        }
    }
    switch (gcd_groups) {
        case 8: Q4_RING2(false, 16);
        case 4: Q4_RING2(false, 8);
        case 2: Q4_RING2(false, 4);
        default: Q4_RING2(false, 2);
    }
#undef Q4_RING2
}

}  // namespace

cudaError_t take_gemv2_error(unsigned int* out) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_gemv2_error, sizeof(unsigned int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_gemv2_error, &zero, sizeof(unsigned int));
    return e;
}

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
    if (dev.smem_optin >= 64 * 1024) {
        const cudaError_t r = launch_gemv2_ring(codes, scales, cb, x, y, N, K, s, dev);
        if (r != cudaErrorNotSupported) return r;
        (void)cudaGetLastError();
    }
    // rows too long for the ring's shared-memory layout: per-lane loads, y
    // zeroed and then added into
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

Q4_DEFINE_TAKE_BOUNDS(gemv2)

}  // namespace q4
