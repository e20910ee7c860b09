// q4_gemm_small.cu -- q4_gemm for M = 2..32 tokens (verify batches, short
// prefill chunks) on sm_100a; q4_gemm sends it M <= 24 (above that the
// two-strip tensor-core kernel streams faster).
//
// What it computes: y[m][n] = sum_g scale[n][g] * sum_{k in g} cb[code(n,k)] * x[m][k]
// ("deep-fold", "Method": 64-weight groups, four-bit codes, one FP16 scale,
// values rebuilt while multiplying; "Trapetum" overview, "What it does": the
// few drafted tokens of speculative decoding are checked in one pass), with
// exact binary16 products and fp32 sums, as the M = 1 kernel.
//
// Why this shape.  Up to 32 tokens the work is still a weight stream (under
// 120 flop per byte), so the kernel is organised around reading each weight
// once at HBM speed and decoding it once for all tokens.
//  * A CTA takes blocks of 128 weight rows over one range of K.  Each of its
//    8 consumer warps owns 16 of the rows for the whole range, so a row's
//    partial sums never leave its warp's registers (no reduction between
//    warps, no shared-memory atomics).
//  * A producer warp streams a block as stages of 128 rows x 512 k: two TMA
//    boxes of 128 rows x 128 code bytes with the 128-byte swizzle, 32 KB per
//    stage, into a 3-stage ring.
//  * Each code byte indexes a byte -> half2 table (cb[lo], cb[hi]) held once
//    per lane in shared memory (entry b of lane l at 256 b + 4 l), so one
//    PRMT forms the address and one LDS returns two rebuilt weights.
//  * The rebuilt weights are the A operand of mma.sync m16n8k16 and the
//    tokens are the columns of B (8 per MMA, one MMA per 8 tokens).
//    Lane (g, tq) reads 8 code bytes of one group of its two rows, so the
//    four k-steps of a group form one MMA chain: the group's fp32 partial sum
//    is scaled by the group's own scale in fp32.
//  * Lane (g, tq) holds rows rho(g) and rho(g) + 8 of its warp's 16 with
//    rho = (0 2 4 6 1 3 5 7): under the 128-byte swizzle the four rows a
//    half-warp reads at once then fall in four different bank windows.
//  * The scales of a stage (8 groups of a row, 16 bytes) arrive by cp.async
//    two stages ahead, into the unused second half of the table's rows, when
//    G is a multiple of 8 (scale rows in 16-byte blocks).  Loads one stage
//    ahead into registers were the top stall (long scoreboard) at M = 8.
//  * x of the CTA's K range is rounded to binary16 once into shared memory,
//    token rows 16 bytes off a multiple of 32 (conflict-free B loads).
//  * K is split across CTAs when x would not fit beside the ring, or when
//    there are too few row blocks to occupy every SM; y is then zeroed first
//    and the partial sums are added with red.global.add.
#include "q4_internal.cuh"
#include "q4_sm100.cuh"

namespace q4 {

__device__ unsigned int g_gemm_small_error;

namespace {

constexpr int kCW = 8;                         // consumer warps
constexpr int kThreads = (kCW + 1) * 32;       // + one producer warp
constexpr int kRows = kCW * 16;                // rows per block
constexpr int kBase = 1024;                    // shared-window address of dynamic shared memory
constexpr int kLutBytes = 65536;               // 256 rows of 256 bytes; lane copies in the first 128
constexpr int kStageK = 512;                   // k per stage
constexpr int kBoxBytes = kRows * 128;         // one TMA box: 128 rows x 128 code bytes
constexpr int kStageBytes = 2 * kBoxBytes;     // 32 KB
constexpr int kNS = 3;                         // ring stages
constexpr uint32_t kRingOff = kLutBytes;
constexpr uint32_t kBarOff = kRingOff + kNS * kStageBytes;
constexpr uint32_t kXOff = kBarOff + 128;
constexpr int kMaxSplits = 64;
constexpr int kXRounds = 8;                    // x chunks in flight per thread in the set-up

struct SmallP {
    const uint16_t* scales;
    const uint16_t* cb;
    const uint16_t* x;
    float* y;
    int M, N, K, G;
    int KR;        // k per split, a multiple of kStageK
    int KS;        // splits of K
    int NB;        // blocks of kRows rows
    int rb_step;   // CTAs per split
    int x_pitch;   // bytes between tokens in the shared-memory copy of x
};

__device__ __forceinline__ uint32_t lut_load(uint32_t off) {
    uint32_t v;
    asm("ld.shared.b32 %0, [%1 + %2];" : "=r"(v) : "r"(off), "n"(kBase));
    return v;
}

template <int kByte>
__device__ __forceinline__ uint32_t lut(uint32_t word, uint32_t lane4) {
    return lut_load(__byte_perm(word, lane4, 0x5504 | (kByte << 4)));
}

// Ring reads stay behind the mbarrier wait that precedes them (volatile).
__device__ __forceinline__ uint2 lds64_ring(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "r"(addr));
    return v;
}

// A read of data another proxy or thread wrote: stays after the wait before it.
__device__ __forceinline__ uint4 lds128_after_wait(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
    uint32_t v;
    asm("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_nc_u16(const void* p) {
    unsigned short v;
    asm("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t cvt_bf16x2_f16x2(uint32_t w) {
    const __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Scales of the 8 groups of stage k range [kb, kb + 512) of one row as four
// binary16 pairs; groups past G repeat a valid one (they multiply x = 0).
template <bool kEvenG>
__device__ __forceinline__ void load_stage_scales(const uint16_t* srow, int kb, int G,
                                                  uint32_t (&out)[4]) {
    const int g0 = kb / kGroup;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (kEvenG) {
            const int g = min(g0 + 2 * i, G - 2);
            out[i] = Q4_IN_BOUNDS(g, 2, G) ? ldg_nc_u32(srow + g) : 0u;
        } else {
            const int ga = min(g0 + 2 * i, G - 1), gb = min(g0 + 2 * i + 1, G - 1);
            out[i] = Q4_IN_BOUNDS(ga, 1, G) && Q4_IN_BOUNDS(gb, 1, G)
                         ? ldg_nc_u16(srow + ga) | (ldg_nc_u16(srow + gb) << 16)
                         : 0u;
        }
    }
}

__device__ __forceinline__ float half_lo(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
}
__device__ __forceinline__ float half_hi(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
}

// Scales of a stage, copied ahead by cp.async into the unused second half of
// the table's 256-byte rows: the 16 bytes (8 groups) of one weight row per
// 16-byte slot; src_bytes < 16 zero-fills the rest (last stage, rows past N).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
constexpr int kScDepth = 3;  // stages of scales in flight per warp

// kAsyncSc (G a multiple of 8): scales come by cp.async two stages ahead into
// shared memory; otherwise by loads one stage ahead into registers.
template <int MB, bool kEvenG, bool kAsyncSc>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_small_kernel(const __grid_constant__ CUtensorMap cmap, const SmallP p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tq = lane & 3;

    const uint32_t base = smem_u32(smem);
    if (base != static_cast<uint32_t>(kBase)) {
        if (tid == 0) atomicOr(&g_gemm_small_error, 0x100u);
        return;
    }
    const uint32_t ring = base + kRingOff;
    const uint32_t bars = base + kBarOff;  // full[kNS], empty[kNS]
    const int split = static_cast<int>(blockIdx.x) % p.KS;
    const int k0 = split * p.KR;
    const int kend = min(p.K, k0 + p.KR);
    const int nst = (kend - k0 + kStageK - 1) / kStageK;  // stages per block
    const int rb_first = static_cast<int>(blockIdx.x) / p.KS;

    if (tid == 0) {
        for (int s = 0; s < kNS; ++s) {
            mbar_init(bars + 8u * s, 1);
            mbar_init(bars + 8u * (kNS + s), kCW);
        }
        fence_mbar_init();
    }
    if (warp == kCW && lane == 0) prefetch_tensor_map(&cmap);
    __syncthreads();

    if (warp == kCW) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            int slot = 0, issued = 0;
            uint32_t eparity = 1;
            bool ok = true;
            for (int rb = rb_first; rb < p.NB && ok; rb += p.rb_step) {
                for (int s = 0; s < nst; ++s) {
                    if (issued >= kNS && !mbar_wait(bars + 8u * (kNS + slot), eparity)) {
                        atomicOr(&g_gemm_small_error, 0x200u);
                        ok = false;
                        break;
                    }
                    const int kb = k0 + s * kStageK;
                    const int nbox = kb + kStageK / 2 < kend ? 2 : 1;
                    const uint32_t dst = ring + slot * kStageBytes;
                    const uint32_t full = bars + 8u * slot;
                    mbar_arrive_expect_tx(full, static_cast<uint32_t>(nbox * kBoxBytes));
                    tma_load_2d(dst, &cmap, kb / 2, rb * kRows, full);
                    if (nbox == 2) tma_load_2d(dst + kBoxBytes, &cmap, kb / 2 + 128, rb * kRows, full);
                    ++issued;
                    if (++slot == kNS) {
                        slot = 0;
                        eparity ^= 1u;
                    }
                }
            }
            // leave once the copies in flight have landed (bounded)
            for (int i = (issued > kNS ? issued - kNS : 0); i < issued; ++i)
                if (!mbar_wait(bars + 8u * (i % kNS), (i / kNS) & 1)) {
                    atomicOr(&g_gemm_small_error, 0x400u);
                    break;
                }
        }
        return;
    }

    // ------------------------------- consumers ------------------------------
    {
        // byte -> (cb[lo], cb[hi]) table, one copy per lane: thread tid writes
        // the 32 copies of entry tid (lane-rotated 16-byte stores)
        static_assert(kCW * 32 == 256, "one table entry per consumer thread");
        const uint32_t ent = static_cast<uint32_t>(p.cb[tid & 15]) |
                             (static_cast<uint32_t>(p.cb[tid >> 4]) << 16);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            *reinterpret_cast<uint4*>(smem + tid * 256 + 16 * ((i + lane) & 7)) =
                make_uint4(ent, ent, ent, ent);
        // x[m][k0, k0 + KR) as binary16, zeros past K
        // (all loads of a batch are issued before the first store: one
        // memory latency per batch of kXRounds chunks per thread)
        const int chunks = p.KR / 8;
        const int total = p.M * chunks;
        for (int i0 = 0; i0 < total; i0 += kXRounds * kCW * 32) {
            uint4 b[kXRounds];
#pragma unroll
            for (int r = 0; r < kXRounds; ++r) {
                const int i = i0 + tid + r * kCW * 32;
                const int m = i / chunks, j = i - m * chunks;
                const int k = k0 + 8 * j;
                b[r] = make_uint4(0u, 0u, 0u, 0u);
                if (i < total && k < p.K &&
                    Q4_IN_BOUNDS(static_cast<int64_t>(m) * p.K + k, 8, static_cast<int64_t>(p.M) * p.K))
                    b[r] = __ldg(reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m) * p.K + k));
            }
#pragma unroll
            for (int r = 0; r < kXRounds; ++r) {
                const int i = i0 + tid + r * kCW * 32;
                if (i < total) {
                    const int m = i / chunks, j = i - m * chunks;
                    uint4 v;
                    v.x = cvt_bf16x2_f16x2(b[r].x);
                    v.y = cvt_bf16x2_f16x2(b[r].y);
                    v.z = cvt_bf16x2_f16x2(b[r].z);
                    v.w = cvt_bf16x2_f16x2(b[r].w);
                    *reinterpret_cast<uint4*>(smem + kXOff + m * p.x_pitch + 16 * j) = v;
                }
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
    }

    const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
    const int rho = (g < 4) ? 2 * g : 2 * (g - 4) + 1;
    const int r1 = 16 * warp + rho;  // this lane's rows in the block: r1, r1 + 8
    const uint32_t row_lo = static_cast<uint32_t>(r1) * 128u;
    const uint32_t row_hi = row_lo + 8u * 128u;
    const uint32_t xlane = base + kXOff + 32u * tq;
    bool bad = false;

    // scales run ahead of the consumer: (nrb, ns) is the cursor of the next
    // stage to fetch
    uint32_t sc_lo[4], sc_hi[4], nx_lo[4], nx_hi[4];
    int nrb = rb_first, ns = 0;
    // kAsyncSc: warp w's slots are table rows 2 kScDepth w + 2 d + h, second
    // half: stage d (mod kScDepth), rows r1 (h = 0) and r1 + 8 (h = 1), slot rho
    const uint32_t sc_slots = base + static_cast<uint32_t>(2 * kScDepth * warp) * 256u + 128u +
                              16u * static_cast<uint32_t>(rho);
    int sc_issued = 0;
    auto fetch_next = [&]() {
        if (nrb < p.NB) {
            if (tq == 0) {
                const int g0 = (k0 + ns * kStageK) / kGroup;
                const uint32_t bytes = static_cast<uint32_t>(min(8, p.G - g0)) * 2u;
                const uint32_t d = static_cast<uint32_t>(sc_issued % kScDepth);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int row = nrb * kRows + r1 + 8 * h;
                    const bool in = row < p.N &&
                                    Q4_IN_BOUNDS(static_cast<int64_t>(row) * p.G + g0, bytes / 2,
                                                 static_cast<int64_t>(p.N) * p.G);
                    cp_async_16(sc_slots + (2u * d + h) * 256u,
                                in ? p.scales + static_cast<int64_t>(row) * p.G + g0 : p.scales,
                                in ? bytes : 0u);
                }
            }
            if (++ns == nst) {
                ns = 0;
                nrb += p.rb_step;
            }
        }
        ++sc_issued;
        cp_async_commit();
    };
    auto load_next = [&]() {
        if (kAsyncSc) {
            fetch_next();
            return;
        }
        if (nrb < p.NB) {
            int n1 = min(nrb * kRows + r1, p.N - 1), n2 = min(nrb * kRows + r1 + 8, p.N - 1);
            const int kb = k0 + ns * kStageK;
            if (!Q4_IN_BOUNDS(n1, 1, p.N) || !Q4_IN_BOUNDS(n2, 1, p.N)) n1 = n2 = 0;
            load_stage_scales<kEvenG>(p.scales + static_cast<int64_t>(n1) * p.G, kb, p.G, nx_lo);
            load_stage_scales<kEvenG>(p.scales + static_cast<int64_t>(n2) * p.G, kb, p.G, nx_hi);
            if (++ns == nst) {
                ns = 0;
                nrb += p.rb_step;
            }
        }
    };
    if (kAsyncSc) fetch_next();  // two stages ahead: stages 0 and 1 now
    load_next();

    int slot = 0;
    uint32_t fparity = 0;
    int sc_used = 0;
    for (int rb = rb_first; rb < p.NB; rb += p.rb_step) {
        float acc[MB][4];
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[mb][q] = 0.f;

        for (int s = 0; s < nst; ++s) {
            if (kAsyncSc) {
                load_next();  // the stage two ahead
                cp_async_wait<kScDepth - 1>();
                __syncwarp();
                const uint32_t d = static_cast<uint32_t>(sc_used % kScDepth);
                const uint4 vl = lds128_after_wait(sc_slots + (2u * d) * 256u);
                const uint4 vh = lds128_after_wait(sc_slots + (2u * d + 1u) * 256u);
                sc_lo[0] = vl.x; sc_lo[1] = vl.y; sc_lo[2] = vl.z; sc_lo[3] = vl.w;
                sc_hi[0] = vh.x; sc_hi[1] = vh.y; sc_hi[2] = vh.z; sc_hi[3] = vh.w;
                ++sc_used;
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    sc_lo[i] = nx_lo[i];
                    sc_hi[i] = nx_hi[i];
                }
                load_next();
            }
            const int kb = k0 + s * kStageK;
            if (!bad && !mbar_wait(bars + 8u * slot, fparity)) {
                bad = true;
                if (lane == 0) atomicOr(&g_gemm_small_error, 0x800u);
            }
            if (!bad) {
                const uint32_t st = ring + slot * kStageBytes;
                // group j of the stage: box j / 4, group j % 4 of the box
                auto group = [&](int j) {
                    const int h = j >> 2, gm = j & 3;
                    const uint32_t box = st + h * kBoxBytes;
                    const int kk = kb + 64 * j;  // first k of the group
                    // 8 code bytes of the group for each row: 16-byte chunk
                    // 2 gm + tq / 2 of the row, swizzled by the row (rho < 8)
                    const uint32_t off =
                        (static_cast<uint32_t>((2 * gm + (tq >> 1)) ^ rho) << 4) + 8u * (tq & 1);
                    const uint2 lo = lds64_ring(box + row_lo + off);
                    const uint2 hi = lds64_ring(box + row_hi + off);
                    // B: x[token][kk + 16 tq, +16) of tokens 8 mb + g
                    uint32_t xb[MB][8];
#pragma unroll
                    for (int mb = 0; mb < MB; ++mb) {
                        const int tok = 8 * mb + g;
                        if (tok < p.M) {
                            const uint32_t a = xlane + tok * p.x_pitch + 2u * (kk - k0);
                            const uint4 v0 = lds128(a), v1 = lds128(a + 16);
                            xb[mb][0] = v0.x; xb[mb][1] = v0.y; xb[mb][2] = v0.z; xb[mb][3] = v0.w;
                            xb[mb][4] = v1.x; xb[mb][5] = v1.y; xb[mb][6] = v1.z; xb[mb][7] = v1.w;
                        } else {
#pragma unroll
                            for (int q = 0; q < 8; ++q) xb[mb][q] = 0u;
                        }
                    }
                    float d[MB][4];
#pragma unroll
                    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                        for (int q = 0; q < 4; ++q) d[mb][q] = 0.f;
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const uint32_t wl = (t < 2) ? lo.x : lo.y;
                        const uint32_t wh = (t < 2) ? hi.x : hi.y;
                        uint32_t a[4];
                        if (t & 1) {
                            a[0] = lut<2>(wl, lane4);
                            a[1] = lut<2>(wh, lane4);
                            a[2] = lut<3>(wl, lane4);
                            a[3] = lut<3>(wh, lane4);
                        } else {
                            a[0] = lut<0>(wl, lane4);
                            a[1] = lut<0>(wh, lane4);
                            a[2] = lut<1>(wl, lane4);
                            a[3] = lut<1>(wh, lane4);
                        }
#pragma unroll
                        for (int mb = 0; mb < MB; ++mb)
                            mma_16816(d[mb], a, xb[mb][2 * t], xb[mb][2 * t + 1], d[mb]);
                    }
                    const float s1 = (j & 1) ? half_hi(sc_lo[j >> 1]) : half_lo(sc_lo[j >> 1]);
                    const float s2 = (j & 1) ? half_hi(sc_hi[j >> 1]) : half_lo(sc_hi[j >> 1]);
#pragma unroll
                    for (int mb = 0; mb < MB; ++mb) {
                        acc[mb][0] = fmaf(s1, d[mb][0], acc[mb][0]);
                        acc[mb][1] = fmaf(s1, d[mb][1], acc[mb][1]);
                        acc[mb][2] = fmaf(s2, d[mb][2], acc[mb][2]);
                        acc[mb][3] = fmaf(s2, d[mb][3], acc[mb][3]);
                    }
                };
                if (kb + kStageK <= kend) {
                    // a full stage: no branch between the groups
#pragma unroll
                    for (int j = 0; j < 8; ++j) group(j);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (kb + 64 * j >= kend) break;
                        group(j);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + 8u * (kNS + slot));
            if (++slot == kNS) {
                slot = 0;
                fparity ^= 1u;
            }
        }
        if (bad) continue;
        // D fragment: rows r1 (q < 2) and r1 + 8, tokens 8 mb + 2 tq + (q & 1)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int m = 8 * mb + 2 * tq + (q & 1);
                const int n = rb * kRows + r1 + 8 * (q >> 1);
                if (m < p.M && n < p.N &&
                    Q4_IN_BOUNDS(static_cast<int64_t>(m) * p.N + n, 1, static_cast<int64_t>(p.M) * p.N)) {
                    float* dst = p.y + static_cast<int64_t>(m) * p.N + n;
                    if (p.KS > 1)
                        red_add_f32(dst, acc[mb][q]);
                    else
                        *dst = acc[mb][q];
                }
            }
    }
    if (kAsyncSc) cp_async_wait<0>();  // no copy outlives the block
}

template <int MB, bool kEvenG, bool kAsyncSc = false>
cudaError_t launch_variant(const CUtensorMap& cmap, const SmallP& p, int grid, int smem, int slot,
                           cudaStream_t s, const DeviceInfo& dev) {
    auto kern = gemm_small_kernel<MB, kEvenG, kAsyncSc>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem, slot, dev.device);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, s>>>(cmap, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t take_gemm_small_error(unsigned int* out) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_gemm_small_error, sizeof(unsigned int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_gemm_small_error, &zero, sizeof(unsigned int));
    return e;
}

cudaError_t launch_gemm_small(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                              const uint16_t* x, float* y, int M, int64_t N, int64_t K,
                              cudaStream_t s, const DeviceInfo& dev) {
    if (M < 2 || M > 32 || dev.smem_reserved != kBase) return cudaErrorNotSupported;
    SmallP p{};
    p.scales = scales;
    p.cb = cb;
    p.x = x;
    p.y = y;
    p.M = M;
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.G = static_cast<int>(K / kGroup);
    p.NB = static_cast<int>((N + kRows - 1) / kRows);

    // x budget: what the table, the ring and the barriers leave
    const int xbudget = dev.smem_optin - static_cast<int>(kXOff);
    const int kstages = static_cast<int>((K + kStageK - 1) / kStageK);
    // Split K: the fewest stages per CTA (the busiest CTA's blocks times the
    // stages of a block, plus a quarter stage of per-block cost); ties go to
    // fewer splits (fewer atomic adds).
    int best_ks = 0, best_grid = 0;
    double best_cost = 0.0;
    for (int ks = 1; ks <= kMaxSplits && ks <= kstages; ++ks) {
        const int kr_stages = (kstages + ks - 1) / ks;
        const int kr = kr_stages * kStageK;
        const int splits = (kstages + kr_stages - 1) / kr_stages;
        if (splits != ks) continue;  // the same split as a smaller ks
        if (M * (2 * kr + 16) > xbudget) continue;
        const int per_split = dev.sm_count / splits;
        if (per_split < 1) break;
        const int rb_step = per_split < p.NB ? per_split : p.NB;
        const int blocks = (p.NB + rb_step - 1) / rb_step;
        const double cost = blocks * (kr_stages + 0.25);
        if (best_ks == 0 || cost < best_cost - 1e-9) {
            best_ks = ks;
            best_cost = cost;
            best_grid = rb_step * splits;
            p.KR = kr;
            p.rb_step = rb_step;
        }
    }
    if (best_ks == 0) return cudaErrorNotSupported;
    p.KS = best_ks;
    p.x_pitch = 2 * p.KR + 16;
    const int smem = static_cast<int>(kXOff) + M * p.x_pitch;

    CUtensorMap cmap;
    cudaError_t e = encode_tensor_map_2d(&cmap, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                                         static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2),
                                         static_cast<uint64_t>(K / 2), kRows, 128,
                                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return cudaErrorNotSupported;  // the caller's fallback kernel runs
    if (p.KS > 1) {
        e = cudaMemsetAsync(y, 0, static_cast<size_t>(M) * static_cast<size_t>(N) * sizeof(float), s);
        if (e != cudaSuccess) return e;
    }
    const bool even = (p.G & 1) == 0;
    if (p.G % 8 == 0) {  // scale rows in 16-byte blocks: cp.async ahead
        if (M <= 8) return launch_variant<1, true, true>(cmap, p, best_grid, smem, 70, s, dev);
        if (M <= 16) return launch_variant<2, true, true>(cmap, p, best_grid, smem, 71, s, dev);
        if (M <= 24) return launch_variant<3, true, true>(cmap, p, best_grid, smem, 72, s, dev);
        return launch_variant<4, true, true>(cmap, p, best_grid, smem, 73, s, dev);
    }
    if (M <= 8)
        return even ? launch_variant<1, true>(cmap, p, best_grid, smem, 40, s, dev)
                    : launch_variant<1, false>(cmap, p, best_grid, smem, 41, s, dev);
    if (M <= 16)
        return even ? launch_variant<2, true>(cmap, p, best_grid, smem, 42, s, dev)
                    : launch_variant<2, false>(cmap, p, best_grid, smem, 43, s, dev);
    if (M <= 24)
        return even ? launch_variant<3, true>(cmap, p, best_grid, smem, 44, s, dev)
                    : launch_variant<3, false>(cmap, p, best_grid, smem, 45, s, dev);
    return even ? launch_variant<4, true>(cmap, p, best_grid, smem, 46, s, dev)
                : launch_variant<4, false>(cmap, p, best_grid, smem, 47, s, dev);
}

Q4_DEFINE_TAKE_BOUNDS(gemm_small)

}  // namespace q4
