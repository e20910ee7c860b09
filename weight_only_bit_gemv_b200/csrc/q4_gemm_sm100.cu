// q4_gemm_sm100.cu -- q4_gemm for M > 24 (prompt processing): a tcgen05
// tensor-core GEMM whose A operand is rebuilt from the 4-bit codes straight
// into tensor memory.
//
// What it computes: y[m][n] = sum_k W[n][k] x[m][k] with W[n][k] =
// cb[code(n,k)] * scale[n][k/64] ("deep-fold", "Method" table: prompt
// processing runs a tensor-core NF4 GEMM that rebuilds weights into
// fragments while it multiplies; no dense weight matrix is written).
//
// Numerics: each weight is rebuilt as binary16(cb * scale) -- HMUL2 of two
// binary16 values, one rounding of the exact product -- and x is rounded to
// binary16 once (exact for 2^-17 <= |x| <= 65504).  Products accumulate in
// fp32 in tensor memory.  The per-weight relative error is at most 2^-11,
// which keeps every output inside 1e-4 * sum|W x| + 1e-6 with a margin of
// ~0.3 sqrt(K) standard deviations (about 20 at K = 4096).
//
// Work: a tile is 128 weight rows (two strips of 128 when BMT <= 128) x BMT
// tokens.  CTAs are persistent, one per SM; each walks its list of segments
// (a run of weight stages of one tile, see SegCursor), the rings below
// running on from one segment to the next.  Roles:
//  * warp 0 streams, by TMA, stages of 4 groups of codes (a 128-row x
//    128-byte box, 128-byte swizzle) with their scales (cp.async);
//  * warp 10 streams, by TMA, the x tile of every group (BMT tokens x 64 k
//    binary16, 128-byte swizzle) into the x stage of the group's ring slot;
//  * warps 2-9 rebuild the weights: thread t of warp w owns row 32 (w mod 4) +
//    t (its tensor-memory lane); per group it reads its 32 code bytes, looks
//    each up in a 256-entry byte -> (cb[lo], cb[hi]) table (one copy per
//    lane), multiplies by the scale with one HMUL2 and writes the 64 weights
//    with one tcgen05.st into the A slot of the group's ring slot.  Even and
//    odd groups go to the two halves of these warps.
//  * warp 1 owns the tensor memory and, per group, issues four tcgen05.mma
//    M=128 N=BMT K=16 (A from tensor memory, B = x tile from shared memory)
//    into one fp32 accumulator of BMT columns, then one commit that frees the
//    group's ring slot (A slot and x stage together); a commit at the end of
//    a segment marks the accumulator ready, and the next segment's first
//    MMA waits until the epilogue has read it out.
//  * warps 2-9, at the start of each segment and after the last, read the
//    previous segment's accumulator (tcgen05.ld) and store it into y (whole
//    tiles) or add it with red.add (parts of a split tile; y zeroed first).
// Measured on B200: with one thread issuing the MMAs, an x stream tied to the
// weight stream and two commits per group, that thread spent most of each
// group waiting for x and committing; the separate x warp and the shared
// ring (one commit) keep the tensor pipe fed.  Each strip re-reads x from L2
// (BMT x 128 bytes per group against 16 KB of codes per 4 groups), and an
// SM takes in only about 50-65 GB/s: with two strips per tile every x tile
// serves 256 rows (both accumulators fit in tensor memory up to BMT = 128),
// which measured 1.2-1.3x faster at M = 40-128.
// Every wait is bounded; a timeout sets an error bit, the roles drain what
// they have in flight and the CTA frees its tensor memory before it exits.
#include <algorithm>
#include <mutex>

#include "q4_internal.cuh"
#include "q4_sm100.cuh"

namespace q4 {

__device__ unsigned int g_gemm_tc_error;

namespace {

constexpr int kR = 128;                   // weight rows per tile = tensor-memory lanes
constexpr int kWG = 4;                    // groups per weight stage
constexpr int kWCodeBytes = kR * 128;     // one code box
constexpr int kWScaleBytes = kR * 8;      // 4 scales per row
constexpr int kLutBytes = 65536;
constexpr int kDecWarps = 8;
constexpr int kXWarp = 2 + kDecWarps;  // the x producer
constexpr int kThreads = (3 + kDecWarps) * 32;
constexpr int kASlots = 4;
constexpr int kWStages = 2;
// The A slots and the x stages form one ring: the MMA warp's one commit per
// group frees both.
constexpr uint32_t kTmemCols = 512;
// Tensor-memory columns: accumulators in [0, 256) (strip h of a two-strip
// tile at column 128 h), A slots in [256, 512): slot s of strip h at
// 256 + 32 (kStrips s + h).
template <int kStrips>
__device__ __forceinline__ uint32_t a_col(int slot, int h) {
    return 256u + 32u * static_cast<uint32_t>(kStrips * slot + h);
}

struct TcGemm {
    const uint16_t* scales;
    const uint16_t* cb;
    float* y;
    int M, N, K, G;
    int BMT;            // tokens per tile (MMA N), multiple of 16, <= 256
    int token_tiles;    // ceil(M / BMT)
    int tiles;          // (strip groups of kStrips strips) x token tiles; tile t = sp * token_tiles + tt
    int W;              // weight stages (kWG groups) per tile: ceil(G / kWG)
    int full;           // stream-K plan: whole tiles per CTA, taken first
    int ks;             // chunk plan (ks >= 1): each tile in ks chunks of cw stages; 0: stream-K plan
    int cw;
    int xstages;
    int xstage_bytes;   // BMT * 128
    int wscale_off, x_off, cb_off, bar_off;
    uint32_t idesc;
};

// The work of one CTA (persistent, one per SM), in order.  Stream-K plan
// (ks == 0): `full` whole tiles (tile i * gridDim.x + blockIdx.x), then an
// even share of the weight stages of the tiles left over: units u over those
// tiles, tile full * gridDim.x + u / W, stage u mod W.  Chunk plan (ks >= 1):
// chunks v = blockIdx.x + i * gridDim.x of the tiles x ks chunks, chunk v
// being stages [cw (v mod ks), +cw) of tile v / ks.  A segment is stages
// [w0, w1) of one tile; it is whole when it covers every stage, and is then
// stored plainly, else added (red.add) into y that the x conversion zeroed.
struct Seg {
    int tile, w0, w1;
};
struct SegCursor {
    int k;
    long long u, u1;
    __device__ explicit SegCursor(const TcGemm& p) : k(0) {
        const long long ru =
            static_cast<long long>(p.tiles - p.full * static_cast<int>(gridDim.x)) * p.W;
        u = ru * blockIdx.x / gridDim.x;
        u1 = ru * (blockIdx.x + 1) / gridDim.x;
    }
    __device__ bool next(const TcGemm& p, Seg& sg) {
        if (p.ks > 0) {
            const long long v = static_cast<long long>(k) * gridDim.x + blockIdx.x;
            if (v >= static_cast<long long>(p.tiles) * p.ks) return false;
            sg.tile = static_cast<int>(v / p.ks);
            sg.w0 = static_cast<int>(v % p.ks) * p.cw;
            sg.w1 = sg.w0 + p.cw < p.W ? sg.w0 + p.cw : p.W;
            ++k;
            return true;
        }
        if (k < p.full) {
            sg.tile = k * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
            sg.w0 = 0;
            sg.w1 = p.W;
            ++k;
            return true;
        }
        if (u >= u1) return false;
        const long long t = u / p.W;
        sg.tile = p.full * static_cast<int>(gridDim.x) + static_cast<int>(t);
        sg.w0 = static_cast<int>(u - t * p.W);
        const long long left = u1 - u;
        sg.w1 = left < p.W - sg.w0 ? sg.w0 + static_cast<int>(left) : p.W;
        u += sg.w1 - sg.w0;
        return true;
    }
};

__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int lane) {
    uint32_t ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity) ? 1u : 0u;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    __syncwarp();
    return ok != 0;
}

template <int kByte>
__device__ __forceinline__ uint32_t lut_at(const uint8_t* smem, uint32_t word, uint32_t lane4) {
    return ld_smem<uint32_t>(smem, __byte_perm(word, lane4, 0x5504 | (kByte << 4)));
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
    return *reinterpret_cast<const uint32_t*>(&r);
}

// kStrips: 128-row strips per tile (2 only with BMT <= 128): both strips
// share every x tile, which halves the x read per weight.
template <bool kAsyncScales, int kStrips>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap xmap,
                   const TcGemm p) {
    constexpr int kStageCode = kStrips * kWCodeBytes;
    constexpr int kStageScale = kStrips * kWScaleBytes;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t base = smem_u32(smem);
    const uint32_t bars = base + p.bar_off;
    // barriers: wfull, wempty [kWStages]; xfull, afull, gdone [kASlots];
    // afilled, cbbar, drain, aempty
    auto wfull = [&](int s) { return bars + 8u * s; };
    auto wempty = [&](int s) { return bars + 8u * (kWStages + s); };
    auto xfull = [&](int s) { return bars + 8u * (2 * kWStages + s); };
    auto afull = [&](int s) { return bars + 8u * (2 * kWStages + kASlots + s); };
    auto gdone = [&](int s) { return bars + 8u * (2 * kWStages + 2 * kASlots + s); };
    const uint32_t afilled = bars + 8u * (2 * kWStages + 3 * kASlots);  // accumulator complete
    const uint32_t cbbar = afilled + 8u;
    const uint32_t drain = afilled + 16u;
    const uint32_t aempty = afilled + 24u;  // accumulator read out by the epilogue
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + p.cb_off + 32);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + p.cb_off + 36);

    if (tid == 0) {
        for (int s = 0; s < kWStages; ++s) {
            mbar_init(wfull(s), 33);  // expect_tx + one arrival per producer lane
            mbar_init(wempty(s), kDecWarps);
        }
        for (int s = 0; s < kASlots; ++s) {
            mbar_init(xfull(s), 1);   // expect_tx
            mbar_init(afull(s), 4);   // the four warps of the owning warpgroup
            mbar_init(gdone(s), 1);   // tcgen05.commit after the group's MMAs
        }
        mbar_init(afilled, 1);
        mbar_init(cbbar, 1);
        mbar_init(drain, 1);
        mbar_init(aempty, kDecWarps);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(base + p.cb_off + 32, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tensor_map(&cmap);
            mbar_arrive_expect_tx(cbbar, 32u);
            bulk_load(base + p.cb_off, p.cb, 32u, cbbar);
        }
        int wi = 0;  // weight stages issued, over all segments
        bool ok = true;
        SegCursor cur(p);
        Seg sg;
        while (ok && cur.next(p, sg)) {
            const int strip = kStrips * (sg.tile / p.token_tiles);
            for (int w = sg.w0; w < sg.w1; ++w, ++wi) {
                // weight stage w of the tile: groups 4w .. min(G, 4w + 4) - 1
                const int ws = wi % kWStages;
                if (wi >= kWStages &&
                    !warp_wait(wempty(ws), static_cast<uint32_t>(wi / kWStages - 1) & 1u, lane)) {
                    ok = false;
                    break;
                }
                const int g0 = kWG * w;
                const int g_end = min(p.G, g0 + kWG);
                const uint32_t cdst = base + kLutBytes + ws * kStageCode;
                const uint32_t sdst = base + p.wscale_off + ws * kStageScale;
                if (lane == 0) {
                    mbar_arrive_expect_tx(wfull(ws), kStageCode);
#pragma unroll
                    for (int h = 0; h < kStrips; ++h)
                        tma_load_2d(cdst + h * kWCodeBytes, &cmap, g0 * 32, (strip + h) * kR, wfull(ws));
                }
#pragma unroll
                for (int jr = 0; jr < kStrips * kR / 32; ++jr) {
                    const int r = lane + 32 * jr;
                    const int row = strip * kR + r;
                    if (kAsyncScales) {
                        const bool in = row < p.N && Q4_IN_BOUNDS(static_cast<long long>(row) * p.G + g0, 4,
                                                                  static_cast<long long>(p.N) * p.G);
                        const uint16_t* src = in ? p.scales + static_cast<long long>(row) * p.G + g0 : p.scales;
                        cp_async_8(sdst + r * 8, src, in ? 8u : 0u);
                    } else {
#pragma unroll
                        for (int q = 0; q < kWG; ++q) {
                            uint16_t v = 0;
                            if (row < p.N && g0 + q < g_end &&
                                Q4_IN_BOUNDS(static_cast<long long>(row) * p.G + g0 + q, 1,
                                             static_cast<long long>(p.N) * p.G))
                                v = p.scales[static_cast<long long>(row) * p.G + g0 + q];
                            sts_u16(sdst + r * 8 + 2 * q, v);
                        }
                    }
                }
                if (kAsyncScales)
                    cp_async_arrive_noinc(wfull(ws));
                else
                    mbar_arrive(wfull(ws));
            }
        }
        if (!ok && lane == 0) {
            atomicOr(&g_gemm_tc_error, 1u);
            *abort_flag = 1;
        }
        // leave only once every copy issued has landed (bounded)
        for (int i = (wi > kWStages ? wi - kWStages : 0); i < wi; ++i)
            if (!warp_wait(wfull(i % kWStages), static_cast<uint32_t>(i / kWStages) & 1u, lane)) break;
    } else if (warp == kXWarp) {
        // ----------------------------- x producer -----------------------------
        // x tile of the CTA's group gi (counted over all segments) -> ring
        // slot gi mod kASlots, reused once the MMAs of group gi - kASlots are done.
        if (lane == 0) prefetch_tensor_map(&xmap);
        int xi = 0;
        bool ok = true, stop = false;
        SegCursor cur(p);
        Seg sg;
        while (ok && !stop && cur.next(p, sg)) {
            const int tt = sg.tile % p.token_tiles;
            const int g_hi = min(p.G, kWG * sg.w1);
            for (int g = kWG * sg.w0; g < g_hi; ++g, ++xi) {
                const int xs = xi % kASlots;
                if (xi >= kASlots &&
                    !warp_wait(gdone(xs), static_cast<uint32_t>(xi / kASlots - 1) & 1u, lane)) {
                    ok = false;
                    break;
                }
                if (__shfl_sync(0xFFFFFFFFu, *abort_flag, 0)) {
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(xfull(xs), static_cast<uint32_t>(p.xstage_bytes));
                    tma_load_2d(base + p.x_off + xs * p.xstage_bytes, &xmap, g * 64, tt * p.BMT, xfull(xs));
                }
                __syncwarp();
            }
        }
        if (!ok && lane == 0) {
            atomicOr(&g_gemm_tc_error, 4u);
            *abort_flag = 1;
        }
        for (int i = (xi > kASlots ? xi - kASlots : 0); i < xi; ++i)
            if (!warp_wait(xfull(i % kASlots), static_cast<uint32_t>(i / kASlots) & 1u, lane)) break;
    } else if (warp == 1) {
        // -------------------------------- MMA ---------------------------------
        // Per segment: wait until the epilogue has read the accumulator of the
        // previous one, then per group four MMAs (the first overwrites the
        // accumulator), one commit that frees the group's A slot and x stage,
        // and at the end a commit that hands the accumulator to the epilogue.
        if (lane == 0) {
            bool ok = true;
            int gi = 0, si = 0;
            SegCursor cur(p);
            Seg sg;
            while (ok && cur.next(p, sg)) {
                if (si > 0 && !mbar_wait(aempty, static_cast<uint32_t>(si - 1) & 1u)) {
                    ok = false;
                    break;
                }
                const int ng = min(p.G, kWG * sg.w1) - kWG * sg.w0;
                for (int k = 0; k < ng; ++k, ++gi) {
                    const int as = gi % kASlots;
                    if (!mbar_wait(afull(as), static_cast<uint32_t>(gi / kASlots) & 1u) ||
                        !mbar_wait(xfull(as), static_cast<uint32_t>(gi / kASlots) & 1u) || *abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bd = smem_desc_sw128(base + p.x_off + as * p.xstage_bytes, 1024);
#pragma unroll
                    for (int h = 0; h < kStrips; ++h)
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            tc_mma_ts(tmem + 128u * h, tmem + a_col<kStrips>(as, h) + 8 * t, bd + 2 * t,
                                      p.idesc, (k > 0 || t > 0) ? 1u : 0u);
                    tc_commit(gdone(as));  // frees the A slot and the x stage
                }
                if (!ok) break;
                tc_commit(afilled);
                ++si;
            }
            if (!ok) {
                atomicOr(&g_gemm_tc_error, 2u);
                *abort_flag = 1;
            }
            tc_commit(drain);
            if (!mbar_wait(drain, 0u)) atomicOr(&g_gemm_tc_error, 16u);
        }
        __syncwarp();
    } else {
        // ------------------------------ decoders -------------------------------
        const int dw = warp - 2, wg = dw >> 2, q = warp & 3;
        const int row = 32 * q + lane;
        const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
        const uint32_t tlane = tmem + (static_cast<uint32_t>(32 * q) << 16);
        bool ok = warp_wait(cbbar, 0u, lane);
        if (ok) {
            const uint32_t cbv = ld_smem<uint16_t>(smem, p.cb_off + 2 * (lane & 15));
            for (int b = dw; b < 256; b += kDecWarps) {
                const uint32_t lo = __shfl_sync(0xFFFFFFFFu, cbv, b & 15);
                const uint32_t hi = __shfl_sync(0xFFFFFFFFu, cbv, b >> 4);
                *reinterpret_cast<uint32_t*>(smem + b * 256 + lane * 4) = lo | (hi << 16);
            }
        }
        named_sync(2, kDecWarps * 32);  // table ready

        // Epilogue of segment `si`: each warpgroup writes half of the
        // accumulator columns, 8 at a time, in a rolled loop (as fast on B200
        // as a 64-column unrolled body, and a fraction of the code).  Whole
        // tiles are stored, parts of a split tile added.
        auto epilogue = [&](const Seg& e, int si) -> bool {
            if (!warp_wait(afilled, static_cast<uint32_t>(si) & 1u, lane)) return false;
            tc_fence_after();
            const int tt = e.tile % p.token_tiles;
            const int strip = kStrips * (e.tile / p.token_tiles);
            const bool add = !(e.w0 == 0 && e.w1 == p.W);
            const int half = p.BMT / 2;
            const int m_beg = tt * p.BMT + wg * half;
            // columns of this warpgroup that hold tokens < M
            const int c_end = min(half, p.M - m_beg);
            for (int hs = 0; hs < kStrips; ++hs) {
                const int n = (strip + hs) * kR + row;
                const bool row_ok = n < p.N;
                const uint32_t tcol = tlane + 128u * hs + static_cast<uint32_t>(wg * half);
                float* dst0 = p.y + static_cast<long long>(m_beg) * p.N + n;
#pragma unroll 1
                for (int c0 = 0; c0 < c_end; c0 += 8) {
                    uint32_t v[8];
                    tc_ld_x8(tcol + c0, v);
                    tc_wait_ld();
                    float* dst = dst0 + static_cast<long long>(c0) * p.N;
#pragma unroll
                    for (int i = 0; i < 8; ++i, dst += p.N) {
                        if (!row_ok || c0 + i >= c_end ||
                            !Q4_IN_BOUNDS(dst - p.y, 1, static_cast<long long>(p.M) * p.N))
                            continue;
                        if (add)
                            red_add_f32(dst, __uint_as_float(v[i]));
                        else
                            *dst = __uint_as_float(v[i]);
                    }
                }
            }
            // the accumulator may now be overwritten by the next segment's MMAs
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(aempty);
            return true;
        };

        // Stage by stage: warpgroup wg decodes the stage's groups j = wg,
        // wg + 2 into A slots (CTA group index) mod 4; both warpgroups
        // release every stage they waited for.
        int gi = 0, wi = 0, si = 0;
        bool epi_ok = true;
        SegCursor cur(p);
        Seg sg, prev{0, 0, 0};
        while (ok && cur.next(p, sg)) {
            if (si > 0 && !(epi_ok = epilogue(prev, si - 1))) break;
            for (int w = sg.w0; w < sg.w1; ++w, ++wi) {
                const int ws = wi % kWStages;
                if (!warp_wait(wfull(ws), static_cast<uint32_t>(wi / kWStages) & 1u, lane) ||
                    __shfl_sync(0xFFFFFFFFu, *abort_flag, 0)) {
                    ok = false;
                    break;
                }
                const int gs = min(kWG, p.G - kWG * w);  // groups in this stage
                const int r8 = row & 7;
                for (int j = wg; j < gs; j += 2) {
                    const int g = gi + j, as = g % kASlots;
                    if (g >= kASlots &&
                        !warp_wait(gdone(as), static_cast<uint32_t>(g / kASlots - 1) & 1u, lane)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int hs = 0; hs < kStrips; ++hs) {
                        const uint32_t rb = kLutBytes + ws * kStageCode + hs * kWCodeBytes + row * 128;
                        const uint4 c0 = ld_smem<uint4>(smem, rb + (((2 * j) ^ r8) << 4));
                        const uint4 c1 = ld_smem<uint4>(smem, rb + (((2 * j + 1) ^ r8) << 4));
                        const uint32_t sb = ld_smem<uint16_t>(
                            smem, p.wscale_off + ws * kStageScale + hs * kWScaleBytes + row * 8 + 2 * j);
                        const uint32_t s2 = sb | (sb << 16);
                        const uint32_t wd[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                        uint32_t h[32];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            h[4 * i + 0] = hmul2_u32(lut_at<0>(smem, wd[i], lane4), s2);
                            h[4 * i + 1] = hmul2_u32(lut_at<1>(smem, wd[i], lane4), s2);
                            h[4 * i + 2] = hmul2_u32(lut_at<2>(smem, wd[i], lane4), s2);
                            h[4 * i + 3] = hmul2_u32(lut_at<3>(smem, wd[i], lane4), s2);
                        }
                        tc_st_x32(tlane + a_col<kStrips>(as, hs), h);
                    }
                    tc_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(afull(as));
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(wempty(ws));
                gi += gs;
            }
            prev = sg;
            ++si;
        }
        if (ok && epi_ok && si > 0) epi_ok = epilogue(prev, si - 1);
        if (!ok && lane == 0) {
            atomicOr(&g_gemm_tc_error, 8u);
            *abort_flag = 1;
        }
        if (!epi_ok && lane == 0) {
            atomicOr(&g_gemm_tc_error, 32u);
            *abort_flag = 1;
        }
    }

    // -------------------------------- teardown --------------------------------
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// The tiles whose segments are added into y rather than stored: y of tiles
// [first, first + count) is zeroed before the GEMM runs.  Tile t covers rows
// [rows * (t / token_tiles), +rows) and tokens [BMT * (t % token_tiles), +BMT).
struct ZeroTiles {
    float* y;
    int M, N, BMT, token_tiles, rows;
    int first, count;
};

// x -> binary16 (xh_elems: elements the destination array holds), then the
// zeroing of the added tiles' outputs.
__global__ void bf16_to_f16_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ xh, int64_t n8,
                                   int64_t xh_elems, const ZeroTiles z) {
    const int64_t per_tile = static_cast<int64_t>(z.BMT) * z.rows;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < z.count * per_tile;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int t = z.first + static_cast<int>(i / per_tile);
        const int r = static_cast<int>(i % per_tile);
        const int m = (t % z.token_tiles) * z.BMT + r / z.rows;
        const int n = (t / z.token_tiles) * z.rows + r % z.rows;
        if (m < z.M && n < z.N &&
            Q4_IN_BOUNDS(static_cast<int64_t>(m) * z.N + n, 1, static_cast<int64_t>(z.M) * z.N))
            z.y[static_cast<int64_t>(m) * z.N + n] = 0.0f;
    }
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (!Q4_IN_BOUNDS(8 * i, 8, xh_elems)) continue;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(x) + i);
        uint4 h;
        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
        uint32_t out[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const __half2 t = __floats2half2_rn(__uint_as_float(in[q] << 16),
                                                __uint_as_float(in[q] & 0xFFFF0000u));
            out[q] = *reinterpret_cast<const uint32_t*>(&t);
        }
        h.x = out[0];
        h.y = out[1];
        h.z = out[2];
        h.w = out[3];
        reinterpret_cast<uint4*>(xh)[i] = h;
    }
}

}  // namespace

cudaError_t launch_prefill_tc(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                              const uint16_t* x, uint16_t* xh, int64_t xh_elems, float* y, int64_t M,
                              int64_t N, int64_t K, cudaStream_t s, const DeviceInfo& dev) {
    TcGemm p{};
    p.scales = scales;
    p.cb = cb;
    p.y = y;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.G = static_cast<int>(K / kGroup);
    // token tiles of at most 256 (the largest MMA N), balanced, multiples of 16
    p.token_tiles = static_cast<int>((M + 255) / 256);
    p.BMT = static_cast<int>(((M + p.token_tiles - 1) / p.token_tiles + 15) / 16 * 16);
    const int strips = static_cast<int>((N + kR - 1) / kR);
    // two strips per tile share each x tile when both accumulators fit
    // (2 x BMT <= 256 tensor-memory columns)
    const int nstrips = p.BMT <= 128 ? 2 : 1;
    p.tiles = (strips + nstrips - 1) / nstrips * p.token_tiles;
    p.W = (p.G + kWG - 1) / kWG;
    // Persistent CTAs, one per SM at most.  Two kinds of plan: stream-K (each
    // CTA takes `full` whole tiles, then an even share of the stages of the
    // tiles left over) and chunks (each tile cut into ks chunks of K, dealt
    // out round-robin).  The cheaper by a cost model measured on B200 with
    // the Llama-2-70B shapes at 32-512 tokens: a weight stage takes
    // 4 x max(0.42 BMT kStrips / 256, 0.12 kStrips) us, each segment a
    // further 2.5 us plus 5.5 us per 128 KB of its tile's outputs (pipeline
    // restart and epilogue, the MMAs idle meanwhile), zeroing y at ~5 TB/s
    // and red.add at ~4 TB/s.  Stream-K wins when most work is in whole
    // tiles; with fewer tiles than SMs, chunks of equal size usually do.
    const double ts = 4.0 * std::max(0.42 * p.BMT * nstrips / 256.0, 0.12 * nstrips);
    const double tile_bytes = 4.0 * p.BMT * nstrips * kR;
    const double te = 2.5 + 5.5 * tile_bytes / 131072.0;
    const double zbw = 5.0e3, rbw = 4.0e3;  // bytes per ns
    const long long units = static_cast<long long>(p.tiles) * p.W;
    int grid = 1;
    double best = -1.0;
    {
        // stream-K
        long long g64 = units / 2 > 0 ? units / 2 : 1;
        if (g64 > dev.sm_count) g64 = dev.sm_count;
        const int gs = static_cast<int>(g64);
        const int full = p.tiles / gs;
        const long long ru = static_cast<long long>(p.tiles - full * gs) * p.W;
        double worst = 0.0, adds = 0.0;
        for (int c = 0; c < gs; ++c) {
            long long u = ru * c / gs;
            const long long u1 = ru * (c + 1) / gs;
            int segs = 0;
            for (; u < u1; ++segs) {
                const long long w0 = u % p.W;
                u += std::min<long long>(u1 - u, p.W - w0);
            }
            adds += segs;
            const double cost = full * (p.W * ts + te) + (u1 - ru * c / gs) * ts + segs * te;
            worst = std::max(worst, cost);
        }
        const double cost = worst + (p.tiles - full * gs) * tile_bytes / (zbw * 1e3) +
                            adds * tile_bytes / (rbw * 1e3);
        best = cost;
        grid = gs;
        p.full = full;
        p.ks = 0;
        p.cw = 0;
    }
    for (int ks = 1; ks <= 8 && ks <= p.W; ++ks) {
        const int cw = (p.W + ks - 1) / ks;
        if ((p.W + cw - 1) / cw != ks) continue;
        const long long vt = static_cast<long long>(p.tiles) * ks;
        const int gk = static_cast<int>(std::min<long long>(vt, dev.sm_count));
        const long long rounds = (vt + gk - 1) / gk;
        double cost = rounds * (cw * ts + te);
        if (ks > 1) {
            const double ybytes = 4.0 * static_cast<double>(M) * static_cast<double>(N);
            cost += ybytes / (zbw * 1e3) + ks * ybytes / (rbw * 1e3);
        }
        if (cost < best) {
            best = cost;
            grid = gk;
            p.full = 0;
            p.ks = ks;
            p.cw = cw;
        }
    }
    p.xstage_bytes = p.BMT * 128;
    p.idesc = idesc_f16_f32(kR, p.BMT);
    p.wscale_off = kLutBytes + kWStages * nstrips * kWCodeBytes;
    p.x_off = (p.wscale_off + kWStages * nstrips * kWScaleBytes + 1023) & ~1023;
    const int SX = kASlots;  // one x stage per A slot
    p.xstages = SX;
    p.cb_off = p.x_off + SX * p.xstage_bytes;
    p.bar_off = p.cb_off + 64;
    const int nbars = 2 * kWStages + 3 * kASlots + 4;
    const int smem = p.bar_off + nbars * 8;
    if (smem > dev.smem_optin) return cudaErrorNotSupported;

    // x -> binary16 into the scratch buffer
    const int64_t n8 = M * K / 8;
    const int zero_tiles = p.ks == 0 ? p.tiles - p.full * grid : (p.ks > 1 ? p.tiles : 0);
    const int64_t zero_elems =
        zero_tiles == p.tiles ? 0 : static_cast<int64_t>(zero_tiles) * p.BMT * nstrips * kR;
    const int64_t work = n8 > zero_elems ? n8 : zero_elems;
    int cgrid = static_cast<int>((work + 255) / 256);
    if (cgrid > dev.sm_count * 8) cgrid = dev.sm_count * 8;
    cudaError_t e = cudaSuccess;
    ZeroTiles z{};
    z.y = y;
    z.M = p.M;
    z.N = p.N;
    z.BMT = p.BMT;
    z.token_tiles = p.token_tiles;
    z.rows = nstrips * kR;
    // tiles whose segments are added: the leftover tiles of stream-K, every
    // tile of a plan in several chunks.  When that is all of y, one memset
    // (faster than the conversion kernel's scalar stores) zeroes it.
    z.first = p.ks == 0 ? p.full * grid : 0;
    z.count = zero_tiles;
    if (zero_tiles == p.tiles) {
        e = cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * sizeof(float), s);
        if (e != cudaSuccess) return e;
        z.count = 0;
    }
    bf16_to_f16_kernel<<<cgrid, 256, 0, s>>>(x, xh, n8, xh_elems, z);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    CUtensorMap cmap, xmap;
    e = encode_tensor_map_2d(&cmap, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(N),
                             static_cast<uint64_t>(K / 2), static_cast<uint64_t>(K / 2), kR, 128,
                             CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = encode_tensor_map_2d(&xmap, xh, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, static_cast<uint64_t>(M),
                             static_cast<uint64_t>(K), static_cast<uint64_t>(K) * 2, p.BMT, 64,
                             CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const bool async_scales = (p.G % kWG) == 0;
    const void* fn = nstrips == 2
                         ? (async_scales ? reinterpret_cast<const void*>(gemm_tc_kernel<true, 2>)
                                         : reinterpret_cast<const void*>(gemm_tc_kernel<false, 2>))
                         : (async_scales ? reinterpret_cast<const void*>(gemm_tc_kernel<true, 1>)
                                         : reinterpret_cast<const void*>(gemm_tc_kernel<false, 1>));
    e = ensure_smem_attr(fn, smem, 30 + (async_scales ? 0 : 1) + 2 * (nstrips - 1), dev.device);
    if (e != cudaSuccess) return e;
    if (nstrips == 2) {
        if (async_scales)
            gemm_tc_kernel<true, 2><<<grid, kThreads, smem, s>>>(cmap, xmap, p);
        else
            gemm_tc_kernel<false, 2><<<grid, kThreads, smem, s>>>(cmap, xmap, p);
    } else {
        if (async_scales)
            gemm_tc_kernel<true, 1><<<grid, kThreads, smem, s>>>(cmap, xmap, p);
        else
            gemm_tc_kernel<false, 1><<<grid, kThreads, smem, s>>>(cmap, xmap, p);
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// q4_gemm's binary16 copy of x: a fixed device array and an ordering event
// ---------------------------------------------------------------------------
// The tensor-core kernel streams x as binary16 by TMA; q4_gemm converts x into
// this array first.  The array is part of the library's image (every GPU that
// loads the library holds it until the process exits), so q4_gemm allocates
// nothing at run time.  One event per device orders the calls that use it:
// each call makes its stream wait for the previous user's kernels (on
// whatever stream) before it writes the array, and records the event after
// its own GEMM, so calls on different streams never use the array at the same
// time.  Under stream capture the wait and the record become external event
// nodes of the graph, so graph replays are ordered the same way.  Inputs
// whose binary16 copy is larger than the array run in chunks of tokens.
// (Converting x inside the kernel instead measured 1.5-1.8x slower at 256 and
// 512 tokens on B200: the conversion doubles the shared-memory traffic of the
// x tiles, and that traffic already bounds the 256-token tile.)
static __device__ __align__(256) uint16_t g_gemm_x[kGemmXBytes / sizeof(uint16_t)];

namespace {
struct GemmXScratch {
    uint16_t* addr = nullptr;
    cudaEvent_t last = nullptr;  // recorded after the latest GEMM that read the array
};
std::mutex g_gemm_x_mu;  // also makes each call's wait / launch / record sequence atomic
GemmXScratch g_gemm_x_dev[64];

// The array's device address and the device's event, set up on first use
// with `device` current.
cudaError_t gemm_x_scratch(int device, GemmXScratch** out) {
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    GemmXScratch& sc = g_gemm_x_dev[device];
    if (!sc.addr) {
        void* a = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&a, g_gemm_x);
        if (e != cudaSuccess) return e;
        e = cudaEventCreateWithFlags(&sc.last, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
        sc.addr = static_cast<uint16_t*>(a);
    }
    *out = &sc;
    return cudaSuccess;
}
}  // namespace

cudaError_t take_gemm_tc_error(unsigned int* out) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_gemm_tc_error, sizeof(unsigned int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_gemm_tc_error, &zero, sizeof(unsigned int));
    return e;
}

cudaError_t prepare_prefill(const DeviceInfo& dev) {
    std::lock_guard<std::mutex> lock(g_gemm_x_mu);
    GemmXScratch* sc = nullptr;
    return gemm_x_scratch(dev.device, &sc);
}

cudaError_t launch_prefill(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                           const uint16_t* x, float* y, int64_t M, int64_t N, int64_t K,
                           cudaStream_t s, const DeviceInfo& dev) {
    std::lock_guard<std::mutex> lock(g_gemm_x_mu);
    GemmXScratch* sc = nullptr;
    cudaError_t e = gemm_x_scratch(dev.device, &sc);
    if (e != cudaSuccess) return e;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(s, &cs);
    if (e != cudaSuccess) return e;
    const bool capturing = cs != cudaStreamCaptureStatusNone;
    // tokens per chunk: as many as the array holds, balanced over the chunks
    const int64_t cap = static_cast<int64_t>(kGemmXBytes / (2 * static_cast<size_t>(K)));
    const int64_t chunks = (M + cap - 1) / cap;
    const int64_t per = (M + chunks - 1) / chunks;
    for (int64_t m0 = 0; m0 < M; m0 += per) {
        const int64_t mc = M - m0 < per ? M - m0 : per;
        e = cudaStreamWaitEvent(s, sc->last, capturing ? cudaEventWaitExternal : cudaEventWaitDefault);
        if (e != cudaSuccess) return e;
        e = launch_prefill_tc(codes, scales, cb, x + m0 * K, sc->addr, kGemmXBytes / 2, y + m0 * N, mc, N,
                              K, s, dev);
        if (e != cudaSuccess) return e;
        e = capturing ? cudaEventRecordWithFlags(sc->last, s, cudaEventRecordExternal)
                      : cudaEventRecord(sc->last, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// ---------------------------------------------------------------------------
// q4_gemm_noalloc: the same tensor-core path with its x scratch in a fixed
// device array instead of the pool, for callers that may not allocate.
// ---------------------------------------------------------------------------
// Every GPU that loads the library holds this array until the process exits.
// All calls share it and it keeps the last call's contents; the conversion
// kernel overwrites the M * K elements a call reads before the GEMM reads
// them, so nothing in it has to start at zero.  Calls whose work overlaps on
// the GPU (other streams, other host threads) race on it.
static __device__ __align__(256) uint16_t g_noalloc_x[Q4_NOALLOC_SCRATCH_BYTES / sizeof(uint16_t)];

// Device address of g_noalloc_x on `device`, which must be current.  Looked
// up once per device; in host code the array's name is only a stand-in.
static cudaError_t noalloc_scratch(int device, uint16_t** out) {
    static std::mutex mu;
    static uint16_t* addr[64] = {};
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[device]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_x);
        if (e != cudaSuccess) return e;
        addr[device] = static_cast<uint16_t*>(p);
    }
    *out = addr[device];
    return cudaSuccess;
}

cudaError_t launch_prefill_noalloc(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                                   const uint16_t* x, float* y, int64_t M, int64_t N, int64_t K,
                                   cudaStream_t s, const DeviceInfo& dev) {
    if (static_cast<uint64_t>(M) * static_cast<uint64_t>(K) * sizeof(uint16_t) > Q4_NOALLOC_SCRATCH_BYTES)
        return cudaErrorInvalidValue;  // rejected earlier by q4_gemm_noalloc
    uint16_t* xh = nullptr;
    const cudaError_t e = noalloc_scratch(dev.device, &xh);
    if (e != cudaSuccess) return e;
    return launch_prefill_tc(codes, scales, cb, x, xh, Q4_NOALLOC_SCRATCH_BYTES / 2, y, M, N, K, s, dev);
}

Q4_DEFINE_TAKE_BOUNDS(gemm_tc)

}  // namespace q4
