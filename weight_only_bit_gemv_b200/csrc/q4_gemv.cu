// q4_gemv.cu -- fused 4-bit codebook GEMV / small-M GEMM for sm_100a, M <= 16.
//
// What it computes: y[m][n] = sum_g scale[n][g] * sum_{k in g} cb[code(n,k)] * x[m][k]
// ("deep-fold", "Method": 64-weight groups with four-bit codes and one FP16
// scale; the decode GEMV rebuilds values while it multiplies and never writes
// a dense matrix; "Trapetum" overview, "What it does": the kernel decodes
// each weight from the codebook as it multiplies).
//
// Design (HBM-bound: 0.53125 bytes per weight must stream at full bandwidth):
//  * Code bytes are decoded through a 256-entry byte -> half2 table in shared
//    memory, (cb[lo nibble], cb[hi nibble]), replicated once per lane so that
//    the 32 lanes of a warp always hit 32 different banks.  Entry b of lane l
//    sits at byte b * 256 + 4 l, so one PRMT builds the address from the code
//    word and one LDS returns two rebuilt weights.
//  * The rebuilt binary16 weights feed mma.sync m16n8k16 as the A operand
//    (16 weight rows x 16 k); x, rounded to binary16, is the B operand (k x 8
//    tokens).  binary16 x binary16 products are exact and the tensor core
//    accumulates in fp32.  The tensor core does the multiply-adds; the SM's
//    issue slots only decode.
//  * The order of k inside an MMA is free, so each lane loads 8 contiguous
//    code bytes of one group of one row (rows g and g+8 of the tile), and MMA t
//    of the group takes bytes 2t, 2t+1 from every lane.  One MMA chain covers
//    exactly one group, so the group's fp32 partial sum is multiplied by the
//    group's scale in fp32 (no rounding of codebook * scale).
//  * A CTA owns a block of 16*RT rows; its 8 warps split the K groups and the
//    partial sums meet in shared memory.  CTAs are persistent over row blocks
//    (grid <= 2 per SM) so the table is built once per CTA.  Codes and scales
//    of the next batch of groups are loaded while the current batch decodes.
//  * x is converted to binary16 once per CTA into shared memory (in K chunks
//    when it does not fit); lanes whose token m >= M load nothing.
#include "q4_internal.cuh"

namespace q4 {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kLutStride = 256;
constexpr int kLutBytes = 256 * kLutStride;
constexpr int kXBudget = 40 * 1024;

struct SmallM {
    const uint8_t* codes;
    const uint16_t* scales;
    const uint16_t* cb;
    const uint16_t* x;
    float* y;
    int M, N, K, G;
    int gc;       // groups per staged x chunk
    int pitch;    // bytes between staged x rows (gc * 128 + 16)
    int x_bytes;  // M * pitch
    int blocks;   // row blocks
};

__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v));
}

__device__ __forceinline__ void sts_u128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w));
}

// bfloat16 pair (lo, hi) -> binary16 pair, round to nearest-even (exact for
// 2^-17 <= |x| <= 65504).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
    const float lo = __uint_as_float(w << 16);
    const float hi = __uint_as_float(w & 0xFFFF0000u);
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Address of table entry (byte `which` of `word`) for this lane: bytes
// [lane*4, code byte, 0, 0] of the table-relative offset.
template <int kByte>
__device__ __forceinline__ uint32_t lut_offset(uint32_t word, uint32_t lane4) {
    return __byte_perm(word, lane4, 0x5504 | (kByte << 4));
}

__device__ void stage_x(const SmallM& p, uint32_t xs, int c0, int cn) {
    const int units_per_row = cn * 8;  // 16-byte units (8 values) per staged row
    const int total = p.M * units_per_row;
    for (int u = threadIdx.x; u < total; u += kThreads) {
        const int m = u / units_per_row;
        const int r = u - m * units_per_row;
        const int64_t off = static_cast<int64_t>(m) * p.K + static_cast<int64_t>(c0) * kGroup + r * 8;
        const uint4 v = Q4_IN_BOUNDS(off, 8, static_cast<int64_t>(p.M) * p.K)
                            ? __ldg(reinterpret_cast<const uint4*>(p.x + off))
                            : make_uint4(0u, 0u, 0u, 0u);
        uint4 h;
        h.x = bf16x2_to_f16x2(v.x);
        h.y = bf16x2_to_f16x2(v.y);
        h.z = bf16x2_to_f16x2(v.z);
        h.w = bf16x2_to_f16x2(v.w);
        sts_u128(xs + m * p.pitch + r * 16, h);
    }
}

template <int RT, int B>
struct Stage {
    uint2 c[B][RT][2];      // code bytes, rows g and g + 8 of each tile
    uint16_t s[B][RT][2];   // binary16 scale bits
};

template <int RT, int B>
__device__ __forceinline__ void load_stage(Stage<RT, B>& st, const SmallM& p, int grp0, int ge,
                                           int r0, int g, int tq) {
    const int64_t rowbytes = p.K / 2;
#pragma unroll
    for (int j = 0; j < B; ++j) {
        const int gj = grp0 + j;
#pragma unroll
        for (int t = 0; t < RT; ++t) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = r0 + 16 * t + g + 8 * h;
                if (gj < ge && row < p.N &&
                    Q4_IN_BOUNDS(row * rowbytes + gj * 32 + tq * 8, 8, p.N * rowbytes) &&
                    Q4_IN_BOUNDS(static_cast<int64_t>(row) * p.G + gj, 1, static_cast<int64_t>(p.N) * p.G)) {
                    st.c[j][t][h] = ldg_stream_u2(p.codes + row * rowbytes + gj * 32 + tq * 8);
                    st.s[j][t][h] = ldg_u16(p.scales + static_cast<int64_t>(row) * p.G + gj);
                } else {
                    st.c[j][t][h] = make_uint2(0u, 0u);
                    st.s[j][t][h] = 0;
                }
            }
        }
    }
}

template <int MB, int RT, int B>
__device__ __forceinline__ void compute_stage(const Stage<RT, B>& st, const SmallM& p, int grp0,
                                              int ge, int c0, const uint8_t* smem, uint32_t lane4,
                                              int g, int tq, float (&acc)[RT][MB][4]) {
#pragma unroll
    for (int j = 0; j < B; ++j) {
        const int gj = grp0 + j;
        if (gj >= ge) break;
        // B operand: x[m][gj*64 + 16 tq .. + 15] as eight binary16 pairs
        uint32_t xb[MB][8];
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) {
            const int m = mb * 8 + g;
            if (m < p.M) {
                const uint32_t a = kLutBytes + m * p.pitch + (gj - c0) * 128 + tq * 32;
                const uint4 v0 = ld_smem<uint4>(smem, a), v1 = ld_smem<uint4>(smem, a + 16);
                xb[mb][0] = v0.x; xb[mb][1] = v0.y; xb[mb][2] = v0.z; xb[mb][3] = v0.w;
                xb[mb][4] = v1.x; xb[mb][5] = v1.y; xb[mb][6] = v1.z; xb[mb][7] = v1.w;
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) xb[mb][q] = 0u;
            }
        }
#pragma unroll
        for (int t = 0; t < RT; ++t) {
            float d[MB][4];
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                for (int q = 0; q < 4; ++q) d[mb][q] = 0.0f;
            const uint2 lo = st.c[j][t][0], hi = st.c[j][t][1];
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
                const uint32_t wl = (tt < 2) ? lo.x : lo.y;
                const uint32_t wh = (tt < 2) ? hi.x : hi.y;
                uint32_t a[4];
                if (tt & 1) {
                    a[0] = ld_smem<uint32_t>(smem, lut_offset<2>(wl, lane4));
                    a[1] = ld_smem<uint32_t>(smem, lut_offset<2>(wh, lane4));
                    a[2] = ld_smem<uint32_t>(smem, lut_offset<3>(wl, lane4));
                    a[3] = ld_smem<uint32_t>(smem, lut_offset<3>(wh, lane4));
                } else {
                    a[0] = ld_smem<uint32_t>(smem, lut_offset<0>(wl, lane4));
                    a[1] = ld_smem<uint32_t>(smem, lut_offset<0>(wh, lane4));
                    a[2] = ld_smem<uint32_t>(smem, lut_offset<1>(wl, lane4));
                    a[3] = ld_smem<uint32_t>(smem, lut_offset<1>(wh, lane4));
                }
#pragma unroll
                for (int mb = 0; mb < MB; ++mb)
                    mma_16816(d[mb], a, xb[mb][2 * tt], xb[mb][2 * tt + 1], d[mb]);
            }
            const float s_lo = __half2float(__ushort_as_half(st.s[j][t][0]));
            const float s_hi = __half2float(__ushort_as_half(st.s[j][t][1]));
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) {
                acc[t][mb][0] = fmaf(s_lo, d[mb][0], acc[t][mb][0]);
                acc[t][mb][1] = fmaf(s_lo, d[mb][1], acc[t][mb][1]);
                acc[t][mb][2] = fmaf(s_hi, d[mb][2], acc[t][mb][2]);
                acc[t][mb][3] = fmaf(s_hi, d[mb][3], acc[t][mb][3]);
            }
        }
    }
}

template <int MB, int RT, int B>
__global__ void __launch_bounds__(kThreads, 2) small_m_kernel(const SmallM p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tq = lane & 3;
    const uint32_t lut = smem_u32(smem);
    const uint32_t xs = lut + kLutBytes;
    float* red = reinterpret_cast<float*>(smem + kLutBytes + p.x_bytes);
    const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;

    // Byte -> (cb[lo], cb[hi]) table, one copy per lane.
    {
        const uint32_t cbv = p.cb[lane & 15];
        for (int b = warp; b < 256; b += kWarps) {
            const uint32_t lo = __shfl_sync(0xFFFFFFFFu, cbv, b & 15);
            const uint32_t hi = __shfl_sync(0xFFFFFFFFu, cbv, b >> 4);
            sts_u32(lut + b * kLutStride + lane4, lo | (hi << 16));
        }
    }

    constexpr int R = RT * 16;
    const int nchunks = (p.G + p.gc - 1) / p.gc;
    for (int blk = blockIdx.x; blk < p.blocks; blk += gridDim.x) {
        const int r0 = blk * R;
        float acc[RT][MB][4];
#pragma unroll
        for (int t = 0; t < RT; ++t)
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[t][mb][q] = 0.0f;

        for (int ch = 0; ch < nchunks; ++ch) {
            const int c0 = ch * p.gc;
            const int cn = min(p.gc, p.G - c0);
            if (nchunks > 1 || blk == static_cast<int>(blockIdx.x)) {
                __syncthreads();
                stage_x(p, xs, c0, cn);
                __syncthreads();
            }
            const int gb = c0 + (warp * cn) / kWarps;
            const int ge = c0 + ((warp + 1) * cn) / kWarps;
            Stage<RT, B> sa, sb;
            int grp = gb;
            if (grp < ge) load_stage(sa, p, grp, ge, r0, g, tq);
            while (grp < ge) {
                if (grp + B < ge) load_stage(sb, p, grp + B, ge, r0, g, tq);
                compute_stage<MB>(sa, p, grp, ge, c0, smem, lane4, g, tq, acc);
                grp += B;
                if (grp >= ge) break;
                if (grp + B < ge) load_stage(sa, p, grp + B, ge, r0, g, tq);
                compute_stage<MB>(sb, p, grp, ge, c0, smem, lane4, g, tq, acc);
                grp += B;
            }
        }

        // Partial sums of the 8 warps meet in shared memory.
#pragma unroll
        for (int t = 0; t < RT; ++t)
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int row = 16 * t + g + 8 * (q >> 1);
                    const int m = mb * 8 + 2 * tq + (q & 1);
                    if (m < p.M) red[(warp * R + row) * p.M + m] = acc[t][mb][q];
                }
        __syncthreads();
        for (int idx = tid; idx < R * p.M; idx += kThreads) {
            const int m = idx / R, row = idx - m * R;
            float sum = 0.0f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) sum += red[(w * R + row) * p.M + m];
            const int n = r0 + row;
            if (n < p.N &&
                Q4_IN_BOUNDS(static_cast<int64_t>(m) * p.N + n, 1, static_cast<int64_t>(p.M) * p.N))
                p.y[static_cast<int64_t>(m) * p.N + n] = sum;
        }
        __syncthreads();
    }
}

template <int MB, int RT, int B>
cudaError_t launch_variant(SmallM p, int slot, cudaStream_t s, const DeviceInfo& dev) {
    const int smem = kLutBytes + p.x_bytes + kWarps * RT * 16 * p.M * 4;
    auto kern = small_m_kernel<MB, RT, B>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem, slot, dev.device);
    if (e != cudaSuccess) return e;
    p.blocks = (p.N + RT * 16 - 1) / (RT * 16);
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const int slots = per_sm * dev.sm_count;
    const int grid = p.blocks < slots ? p.blocks : slots;
    kern<<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_small_m(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                           const uint16_t* x, float* y, int M, int64_t N, int64_t K,
                           cudaStream_t s, const DeviceInfo& dev) {
    if (M <= 4) {
        cudaError_t e = launch_gemv_m1(codes, scales, cb, x, y, M, N, K, s, dev);
        if (e != cudaErrorNotSupported) return e;
        (void)cudaGetLastError();
    }
    if (M >= 2) {
        cudaError_t e = launch_gemm_small(codes, scales, cb, x, y, M, N, K, s, dev);
        if (e != cudaErrorNotSupported) return e;
        (void)cudaGetLastError();
    }
    SmallM p{};
    p.codes = codes;
    p.scales = scales;
    p.cb = cb;
    p.x = x;
    p.y = y;
    p.M = M;
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.G = static_cast<int>(K / kGroup);
    int gc = (kXBudget / M - 16) / 128;
    if (gc > p.G) gc = p.G;
    if (gc < 1) gc = 1;
    p.gc = gc;
    p.pitch = gc * 128 + 16;
    p.x_bytes = M * p.pitch;

    const int64_t tiles = (N + 15) / 16;
    const int64_t slots = 2LL * dev.sm_count;
    if (M <= 8) {
        if (tiles >= 8 * slots) return launch_variant<1, 4, 1>(p, 0, s, dev);
        if (tiles >= 2 * slots) return launch_variant<1, 2, 2>(p, 1, s, dev);
        return launch_variant<1, 1, 4>(p, 2, s, dev);
    }
    if (tiles >= 2 * slots) return launch_variant<2, 2, 2>(p, 3, s, dev);
    return launch_variant<2, 1, 4>(p, 4, s, dev);
}

Q4_DEFINE_TAKE_BOUNDS(gemv)

}  // namespace q4
