// q4_gemv_m1.cu -- the M = 1 decode GEMV on sm_100a.
//
// What it computes: y[n] = sum_g scale[n][g] * sum_{k in g} cb[code(n,k)] * x[k]
// ("deep-fold", "Method": 64-weight groups, four-bit codes, one FP16 scale;
// the decode GEMV rebuilds values while it multiplies and writes no dense
// matrix; "Trapetum" overview, "The bandwidth law": decode time is the time
// to read the weight bytes).
//
// Why this shape.  Decode streams 0.53125 bytes per weight, so the kernel is
// an HBM stream with the decode hidden under it.
//  * DRAM sees long contiguous reads issued as few, large bulk copies.  CTA c
//    owns the rows [N c / grid, N (c + 1) / grid), a contiguous range of the
//    code matrix.  A producer warp copies it into a shared-memory ring with
//    1-D bulk copies (cp.async.bulk), one 16-row tile (or a 16-row x 2 KB
//    slice of it) per stage: a whole tile of rows up to 2 KB long is one
//    contiguous copy, longer rows are copied one ~2 KB row segment at a
//    time.  On B200 a bulk copy costs about 50 ns of its SM's copy engine
//    whatever its size, so copies of 1 KB or less cap the stream far below
//    the HBM rate, and reads of 64-128 bytes of many rows at a time (per-lane
//    loads, 2-D tensor boxes) lose DRAM efficiency; the layout above avoids
//    both.
//  * Each code byte indexes a 256-entry byte -> half2 table (cb[lo nibble],
//    cb[hi nibble]) held once per lane (entry b of lane l at 256 b + 4 l, at
//    the start of dynamic shared memory), so one PRMT of (code word, 4 l)
//    forms the address, the table's shared-window base is an immediate of
//    the load, and the 32 lanes hit 32 banks; one LDS returns two weights.
//  * The weights are the A operand of mma.sync m16n8k16 (binary16 products
//    are exact, sums are fp32).  A warp's unit is 16 rows x 256 k (two spans
//    of 128 k, four groups).  In pass A the even rows of the tile take span
//    2u and the odd rows span 2u + 1; in pass B they swap.  Lane (g, tq) reads
//    16 code bytes of rows g and g + 8, so a quarter warp (rows g, g + 1)
//    always reads 128 distinct bytes (no bank conflicts, no padding).  The B
//    operand's columns 0-3 hold x of the unit's four groups, each zero
//    outside its group, so one chain of eight MMAs per pass yields every
//    row's per-group sums in columns 0-3; lane tq in {0, 1} keeps span
//    2u + tq of its rows and scales each group's fp32 sum by its own scale.
//  * x is rounded to binary16 once per CTA.  When a tile is one stage, each
//    warp loads its units' B fragments straight into registers for the whole
//    kernel; otherwise x goes to shared memory in that column layout (for
//    K <= 8192 inside the unused half of the table rows).  Scales are read
//    from global memory by the consumers, stages ahead.
//  * Each warp stores its tile sums in its own shared-memory slot (no
//    atomics); at the end of a pass of tiles the CTA adds the warps' slots
//    and writes each y element once (no split-K between CTAs, no zeroing of
//    y, no global atomics).
//  * Programmatic dependent launch: the kernel lets the next kernel on the
//    stream launch at once, prefetches the first stages of its weights into
//    L2 (a prefetch only warms the cache, so it never reads stale data), and
//    waits for the preceding kernel before it reads any input.
#include "q4_internal.cuh"
#include "q4_sm100.cuh"

namespace q4 {

__device__ unsigned int g_gemv_m1_error;

namespace {

constexpr int kCW = 16;                   // consumer warps (16 measured 3-5 % faster than 8)
constexpr int kUPW = 1;                   // units per consumer warp per stage
constexpr int kThreads = (kCW + 1) * 32;  // + one producer warp
constexpr int kBase = 1024;               // shared-window address of dynamic shared memory
constexpr int kLutBytes = 65536;          // 256 rows of 256 bytes; lane copies in the first 128
constexpr int kSpan = 128;                // k per span (64 code bytes)
constexpr int kMaxKC = 2048;              // code bytes of a row per stage
constexpr int kMinPassTiles = 8;          // tiles per pass of the per-warp row partials (at least)
constexpr int kMaxPassTiles = 64;
constexpr uint32_t kTileSlotBytes = kCW * 16 * 4;  // one tile's partials of every warp, per token
constexpr int kAhead = 3;                 // scale prefetch distance, in stages
constexpr int kMaxStages = 6;
constexpr int kXEmbedSpans = 64;          // spans whose x fits in the table rows' free halves
constexpr int kXRounds = 13;              // x chunk loads per consumer thread: K <= 13 * 256 * 8
constexpr uint32_t kAccOff = kLutBytes;

static_assert(2 * kMaxStages * 8 <= 128, "barriers overflow their area");

struct M1 {
    const uint8_t* codes;
    const uint16_t* scales;
    const uint16_t* cb;
    const uint16_t* x;
    float* y;
    int M;           // tokens (1..4)
    int N, K, G, S;  // S = spans of 128 k (the last may hold one group)
    int SP;          // S rounded up to even: x holds a zero span S when S is odd
    int rowbytes;    // K / 2
    int KC;          // code bytes of a row per stage (the ring's row pitch)
    int C;           // stages per 16-row tile
    int NS;          // ring stages
    int PT;          // tiles per pass of the row partials
    uint32_t bar_off, x_off;  // barriers (128 bytes), then x when it is not in the table rows
    uint32_t ring_off, stage_bytes;
};

// Scale reads go through L1: the consumer warps read neighbouring pairs of
// the same rows, so most of them hit lines another warp brought in (measured:
// non-allocating scale loads cost a quarter of the kernel's throughput).
__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
    uint32_t v;
    asm("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// A load that stays under the branch that guards it (never hoisted).
__device__ __forceinline__ uint4 ldg_v4_ordered(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_u16(const void* p) {
    unsigned short v;
    asm("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// Table read: `off` is a dynamic-shared-memory offset.
__device__ __forceinline__ uint32_t lds32_dyn(uint32_t off) {
    uint32_t v;
    asm("ld.shared.b32 %0, [%1 + %2];" : "=r"(v) : "r"(off), "n"(kBase));
    return v;
}

template <int kOff>
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4 + %5];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "r"(addr), "n"(kOff));
    return v;
}

// Ring reads stay behind the mbarrier wait that precedes them (volatile).
template <int kOff>
__device__ __forceinline__ uint4 lds128_ring(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4 + %5];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr), "n"(kOff));
    return v;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// The scales of rows [row0, row1) lie contiguously; warm L2 with them (the
// range is shrunk to whole 16-byte blocks inside the buffer).
__device__ __forceinline__ void prefetch_scales_l2(const uint16_t* scales, int64_t G, int64_t N,
                                                   int row0, int row1) {
    const uint64_t b0 = (static_cast<uint64_t>(row0) * G * 2 + 15) & ~15ull;
    const uint64_t b1 = (static_cast<uint64_t>(row1) * G * 2) & ~15ull;
    const uint64_t end = (static_cast<uint64_t>(N) * G * 2) & ~15ull;
    const uint64_t e = b1 < end ? b1 : end;
    if (e > b0)
        prefetch_l2(reinterpret_cast<const uint8_t*>(scales) + b0, static_cast<uint32_t>(e - b0));
}

__device__ __forceinline__ uint32_t cvt_bf16x2_f16x2(uint32_t w) {
    const __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float f16_lo(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
}
__device__ __forceinline__ float f16_hi(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
}

// Table entry (cb[lo], cb[hi]) of byte kByte of `word` for this lane: offset
// [lane*4, code byte, 0, 0] from the start of dynamic shared memory.
template <int kByte>
__device__ __forceinline__ uint32_t lut(uint32_t word, uint32_t lane4) {
    return lds32_dyn(__byte_perm(word, lane4, 0x5504 | (kByte << 4)));
}

__device__ __forceinline__ uint32_t lane4_of(int lane) { return static_cast<uint32_t>(lane) * 4u; }

// One pass over the 128 k of this lane's row slots: eight MMAs per token
// pair in two independent chains of four (the sums of k-steps 0-3 and 4-7),
// so that a warp keeps more MMAs in flight; the rebuilt weights serve every
// pair.
template <int MP>
__device__ __forceinline__ void pass_mma(uint4 lo, uint4 hi, const uint32_t (&xr)[MP][16],
                                         uint32_t lane4, float (&d)[MP][4], float (&e)[MP][4]) {
    const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w};
    const uint32_t wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const uint32_t l = wl[t >> 1], h = wh[t >> 1];
        uint32_t a[4];
        if (t & 1) {
            a[0] = lut<2>(l, lane4);
            a[1] = lut<2>(h, lane4);
            a[2] = lut<3>(l, lane4);
            a[3] = lut<3>(h, lane4);
        } else {
            a[0] = lut<0>(l, lane4);
            a[1] = lut<0>(h, lane4);
            a[2] = lut<1>(l, lane4);
            a[3] = lut<1>(h, lane4);
        }
#pragma unroll
        for (int pp = 0; pp < MP; ++pp) {
            if (t < 4)
                mma_16816(d[pp], a, xr[pp][2 * t], xr[pp][2 * t + 1], d[pp]);
            else
                mma_16816(e[pp], a, xr[pp][2 * t], xr[pp][2 * t + 1], e[pp]);
        }
    }
}

// Scales of groups 2s, 2s + 1 of a row (`srow` = its first scale) as a
// binary16 pair; the second repeats the first when 2s + 1 == G (it then
// multiplies a zero sum).
template <bool kEvenG>
__device__ __forceinline__ uint32_t load_scales(const M1& p, const uint16_t* srow, int s) {
    const uint16_t* q = srow + 2 * s;
    [[maybe_unused]] const long long extent = static_cast<long long>(p.N) * p.G;
    if (kEvenG) return Q4_IN_BOUNDS(q - p.scales, 2, extent) ? ldg_u32(q) : 0u;
    const uint16_t* q1 = q + (2 * s + 1 < p.G ? 1 : 0);
    if (!Q4_IN_BOUNDS(q - p.scales, 1, extent) || !Q4_IN_BOUNDS(q1 - p.scales, 1, extent)) return 0u;
    return ldg_u16(q) | (ldg_u16(q1) << 16);
}

// MT: token slots (1, 2 or 4); tokens 2 pp and 2 pp + 1 share B operand pp.
template <bool kEvenG, bool kWhole, bool kXEmb, int MT>
__global__ void __launch_bounds__(kThreads, 1) gemv_m1_kernel(const M1 p) {
    static_assert(MT == 1 || ((MT == 2 || MT == 4) && kWhole), "several tokens only with whole rows");
    constexpr int MP = (MT + 1) / 2;  // B operands (token pairs)
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tq = lane & 3;

    // The next kernel on the stream may launch now; it waits for this one
    // before it reads anything this one writes.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // Table reads use the dynamic-shared-memory base as an immediate; a
    // different base is reported (bit 8 of q4_timeout_flags) instead of used.
    const uint32_t base = smem_u32(smem);
    if (base != static_cast<uint32_t>(kBase)) {
        if (tid == 0) atomicOr(&g_gemv_m1_error, 0x100u);
        return;
    }
    const uint32_t bars = base + p.bar_off;
    const int NS = p.NS;
    const int r0 = static_cast<int>(static_cast<int64_t>(p.N) * blockIdx.x / gridDim.x);
    const int r1 = static_cast<int>(static_cast<int64_t>(p.N) * (blockIdx.x + 1) / gridDim.x);
    const int nrows = r1 - r0;
    const int T = (nrows + 15) >> 4;
    const int total = T * p.C;  // stages of this CTA

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bars + 8u * s, 1);           // full: the producer's expect_tx
            mbar_init(bars + 8u * (NS + s), kCW);  // empty: one arrival per consumer warp
        }
        fence_mbar_init();
    }
    // x may be written by the preceding kernel: before the wait it is only
    // prefetched into L2 (a prefetch is coherent, L2 being the point of
    // coherence), so the reads after the wait find it there.
    if (warp == kCW && lane == 30) prefetch_l2(p.x, static_cast<uint32_t>(p.K) * 2u);
    // Warm L2 with the first stage and its scales while the preceding kernel
    // finishes (more would queue ahead of the reads of x).
    if (warp == kCW && total > 0) {
        const int rows = min(16, nrows);
        if (kWhole) {
            if (lane == 0)
                prefetch_l2(p.codes + static_cast<int64_t>(r0) * p.rowbytes,
                            static_cast<uint32_t>(rows * p.rowbytes));
        } else if (lane < rows) {
            prefetch_l2(p.codes + static_cast<int64_t>(r0 + lane) * p.rowbytes,
                        static_cast<uint32_t>(min(p.KC, p.rowbytes)));
        }
    }
    if (warp == kCW && lane == 31) prefetch_scales_l2(p.scales, p.G, p.N, r0, r0 + min(nrows, 32));
    if (warp == kCW && lane == 29) prefetch_l2(p.cb, 32u);
    __syncthreads();

    if (warp == kCW) {
        // ------------------------------ producer ------------------------------
        const uint32_t ring = base + p.ring_off;
        int slot = 0, t = 0, c = 0;
        uint32_t eparity = 1;  // parity of the empty phase to wait for (round - 1)
        auto issue = [&]() {
            const int rows = min(16, nrows - 16 * t);
            const uint32_t dst = ring + slot * p.stage_bytes;
            const uint32_t full = bars + 8u * slot;
            // The consumers read scales with small loads; have the tile two
            // ahead's scales in L2 by then (one contiguous block per tile).
            if (c == 0 && lane == 31 && 16 * (t + 2) < nrows)
                prefetch_scales_l2(p.scales, p.G, p.N, r0 + 16 * (t + 2),
                                   r0 + min(nrows, 16 * (t + 3)));
            if (kWhole) {
                if (lane == 0) {
                    const uint32_t bytes = static_cast<uint32_t>(rows * p.rowbytes);
                    mbar_arrive_expect_tx(full, bytes);
                    if (Q4_IN_BOUNDS(static_cast<int64_t>(r0 + 16 * t) * p.rowbytes, bytes,
                                     static_cast<int64_t>(p.N) * p.rowbytes))
                        bulk_load(dst, p.codes + static_cast<int64_t>(r0 + 16 * t) * p.rowbytes, bytes,
                                  full);
                }
            } else {
                const uint32_t bytes = static_cast<uint32_t>(min(p.KC, p.rowbytes - c * p.KC));
                if (lane == 0) mbar_arrive_expect_tx(full, bytes * rows);
                __syncwarp();
                if (lane < rows &&
                    Q4_IN_BOUNDS(static_cast<int64_t>(r0 + 16 * t + lane) * p.rowbytes + c * p.KC, bytes,
                                 static_cast<int64_t>(p.N) * p.rowbytes))
                    bulk_load(dst + lane * p.KC,
                              p.codes + static_cast<int64_t>(r0 + 16 * t + lane) * p.rowbytes +
                                  c * p.KC,
                              bytes, full);
            }
            if (++c == p.C) {
                c = 0;
                ++t;
            }
            if (++slot == NS) {
                slot = 0;
                eparity ^= 1u;
            }
        };
        // The set-up's reads of x and the codebook go out first; the weight
        // stream starts once every consumer has issued them.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        asm volatile("bar.sync 2, %0;" ::"n"(kThreads) : "memory");
        for (int i = 0; i < total; ++i) {
            if (i == 2) {
                // let the first stage land before the rest of the ring is
                // requested, so that it is not served behind them
                uint32_t ok = 1;
                if (lane == 0) ok = mbar_wait(bars, 0u) ? 1u : 0u;
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) {
                    if (lane == 0) atomicOr(&g_gemv_m1_error, 0x200u);
                    break;
                }
            }
            if (i >= NS) {
                uint32_t ok = 1;
                if (lane == 0) ok = mbar_wait(bars + 8u * (NS + slot), eparity) ? 1u : 0u;
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) {
                    if (lane == 0) atomicOr(&g_gemv_m1_error, 0x200u);
                    break;
                }
            }
            issue();
        }
        // Leave only once this warp's copies have landed (bounded).
        if (lane == 0) {
            for (int i = (total > NS ? total - NS : 0); i < total; ++i)
                if (!mbar_wait(bars + 8u * (i % NS), (i / NS) & 1)) {
                    atomicOr(&g_gemv_m1_error, 0x400u);
                    break;
                }
        }
        return;
    }

    // ------------------------------- consumers ------------------------------
    float* acc_s = reinterpret_cast<float*>(smem + kAccOff);
    constexpr uint32_t kXSpan = kXEmb ? 1024u : 512u;  // x bytes between spans
    const int upk = p.KC >> 7;                         // units (256 k) per full stage
    // this lane's code offsets in a stage: rows g and g + 8, pass A and B
    const uint32_t ring_lane = base + p.ring_off + g * p.KC + 16 * tq;
    const uint32_t offA = 64 * (g & 1), offB = 64 - offA;
    const uint32_t rowhi = 8 * p.KC;
    const bool use_a = (tq & 1) == (g & 1);
    bool bad = false;

    // Scales of the stages ahead ([0] = the current stage's): for unit j of
    // this warp, span 2U + (tq & 1) of rows g and g + 8.  The prefetch cursor
    // (st, sc) runs kAhead stages ahead of the consumer's.
    uint32_t sc[kAhead][kUPW][2];
    int st = 0, scc = 0, sleft = total;
    const uint16_t* srow_lo = nullptr;
    const uint16_t* srow_hi = nullptr;
    auto scale_rows = [&]() {
        srow_lo = p.scales + static_cast<int64_t>(r0 + min(16 * st + g, nrows - 1)) * p.G;
        srow_hi = p.scales + static_cast<int64_t>(r0 + min(16 * st + g + 8, nrows - 1)) * p.G;
    };
    int soff[kUPW];  // whole rows: the span of unit j never changes
#pragma unroll
    for (int j = 0; j < kUPW; ++j) soff[j] = min(2 * (warp + kCW * j) + (tq & 1), p.S - 1);
    auto next_scales = [&](uint32_t (&out)[kUPW][2]) {
#pragma unroll
        for (int j = 0; j < kUPW; ++j) out[j][0] = out[j][1] = 0u;
        if (kWhole) {
            if (sleft > 0) {
#pragma unroll
                for (int j = 0; j < kUPW; ++j) {
                    out[j][0] = load_scales<kEvenG>(p, srow_lo, soff[j]);
                    out[j][1] = load_scales<kEvenG>(p, srow_hi, soff[j]);
                }
                --sleft;
                ++st;
                scale_rows();
            }
        } else if (sleft > 0) {
#pragma unroll
            for (int j = 0; j < kUPW; ++j) {
                const int sp = min(2 * (scc * upk + warp + kCW * j) + (tq & 1), p.S - 1);
                out[j][0] = load_scales<kEvenG>(p, srow_lo, sp);
                out[j][1] = load_scales<kEvenG>(p, srow_hi, sp);
            }
            --sleft;
            if (++scc == p.C) {
                scc = 0;
                ++st;
                scale_rows();
            }
        }
    };

    // this thread's table entry b = tid: (cb[b & 15], cb[b >> 4])

    auto cb_entry = [&]() -> uint32_t {
        return static_cast<uint32_t>(p.cb[tid & 15]) | (static_cast<uint32_t>(p.cb[(tid >> 4) & 15]) << 16);
    };
    // byte -> (cb[lo], cb[hi]) table, one copy per lane: thread tid writes the
    // 32 copies of entry tid, four per 16-byte store, starting at a
    // lane-rotated chunk so that a store of the warp spreads over the banks
    auto build_table = [&](uint32_t ent) {
#pragma unroll
        for (int i = 4 * (tid >> 8); i < 4 * (tid >> 8) + 4; ++i)
            *reinterpret_cast<uint4*>(smem + (tid & 255) * 256 + 16 * ((i + lane) & 7)) =
                make_uint4(ent, ent, ent, ent);
    };
    uint32_t xw[kUPW][MP][16];  // whole rows: this warp's units never change, nor their x
    asm volatile("griddepcontrol.wait;" ::: "memory");
    {
        // Issue every global read of the set-up at once, then build the table
        // and x: one memory latency instead of one per round.
        const uint32_t ent = cb_entry();
        const int nx = p.K >> 3;  // 16-byte chunks of x (8 values)
        uint4 xv[kXRounds];
        if (kWhole) {
            // The B fragments of this warp's units U = warp + kCW j straight
            // from x, in the column layout the shared-memory copy has
            // otherwise: lane (g, tq) holds x[128 s + 32 tq, +32) of span
            // s = 2 U + (g / 2) % 2 when g % 2 == tq / 2, else zeros.
#pragma unroll
            for (int j = 0; j < kUPW; ++j) {
                const int U = warp + kCW * j;
#pragma unroll
                for (int pp = 0; pp < MP; ++pp) {
                    // B columns 0-3 (lanes g < 4) hold token 2 pp, columns 4-7
                    // token 2 pp + 1
                    const int tok = 2 * pp + (g >> 2);
                    const bool act = U < upk && (g & 1) == (tq >> 1) && tok < p.M;
                    const uint16_t* xs = p.x + static_cast<int64_t>(tok) * p.K +
                                         kSpan * (2 * U + ((g >> 1) & 1)) + 32 * tq;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 v = make_uint4(0u, 0u, 0u, 0u);
                        if (act && Q4_IN_BOUNDS(xs + 8 * q - p.x, 8, static_cast<int64_t>(p.M) * p.K))
                            v = ldg_v4_ordered(xs + 8 * q);
                        xw[j][pp][4 * q] = v.x;
                        xw[j][pp][4 * q + 1] = v.y;
                        xw[j][pp][4 * q + 2] = v.z;
                        xw[j][pp][4 * q + 3] = v.w;
                    }
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < kXRounds; ++i) {
                const int r = tid + i * kCW * 32;
                xv[i] = r < nx && Q4_IN_BOUNDS(8 * r, 8, p.K) ? __ldg(reinterpret_cast<const uint4*>(p.x) + r)
                                                              : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        asm volatile("bar.sync 2, %0;" ::"n"(kThreads) : "memory");
        build_table(ent);
        if (kWhole) {
#pragma unroll
            for (int j = 0; j < kUPW; ++j)
#pragma unroll
                for (int pp = 0; pp < MP; ++pp)
#pragma unroll
                    for (int i = 0; i < 16; ++i) xw[j][pp][i] = cvt_bf16x2_f16x2(xw[j][pp][i]);
        } else {
            // x as binary16: 16-byte chunk (span s, quarter q, parity par, j)
            // holds x[128 s + 32 j + 8 q, +8) when par == j / 2 (the column
            // of that group), else zeros; chunks past K are zeros.
            auto chunk_off = [&](int s, int q, int par, int j) -> uint32_t {
                return kXEmb ? (4 * s + q) * 256 + 128 + par * 64 + j * 16
                             : p.x_off + s * 512 + q * 128 + par * 64 + j * 16;
            };
#pragma unroll
            for (int i = 0; i < kXRounds; ++i) {
                const int r = tid + i * kCW * 32;
                if (r < nx) {
                    const int k = 8 * r;
                    const int s = k >> 7, j = (k >> 5) & 3, q = (k >> 3) & 3;
                    uint4 h;
                    h.x = cvt_bf16x2_f16x2(xv[i].x);
                    h.y = cvt_bf16x2_f16x2(xv[i].y);
                    h.z = cvt_bf16x2_f16x2(xv[i].z);
                    h.w = cvt_bf16x2_f16x2(xv[i].w);
                    *reinterpret_cast<uint4*>(smem + chunk_off(s, q, j >> 1, j)) = h;
                    *reinterpret_cast<uint4*>(smem + chunk_off(s, q, 1 - (j >> 1), j)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
            }
            // the spans that reach past K: their chunks beyond K are zeros
            for (int c = (p.S - 1) * 32 + tid; c < p.SP * 32; c += kCW * 32) {
                const int j = c & 3, par = (c >> 2) & 1, q = (c >> 3) & 3, s = c >> 5;
                if (s * kSpan + 32 * j + 8 * q >= p.K)
                    *reinterpret_cast<uint4*>(smem + chunk_off(s, q, par, j)) =
                        make_uint4(0u, 0u, 0u, 0u);
            }
        }
    }
    scale_rows();
#pragma unroll
    for (int i = 0; i < kAhead; ++i) next_scales(sc[i]);

    // One unit: two passes of eight MMAs per token pair; lane tq adds span
    // 2U + (tq & 1) of rows g and g + 8 (token 2 pp + tq / 2), each group
    // scaled by its own scale.
    auto unit = [&](uint32_t a, const uint32_t (&xr)[MP][16], const uint32_t (&s)[2],
                    float (&acc_lo)[MP], float (&acc_hi)[MP]) {
        const uint4 loA = lds128_ring<0>(a + offA), hiA = lds128_ring<0>(a + offA + rowhi);
        const uint4 loB = lds128_ring<0>(a + offB), hiB = lds128_ring<0>(a + offB + rowhi);
        float dA[MP][4], eA[MP][4], dB[MP][4], eB[MP][4];
#pragma unroll
        for (int pp = 0; pp < MP; ++pp)
#pragma unroll
            for (int i = 0; i < 4; ++i) dA[pp][i] = eA[pp][i] = dB[pp][i] = eB[pp][i] = 0.f;
        pass_mma<MP>(loA, hiA, xr, lane4_of(lane), dA, eA);
        pass_mma<MP>(loB, hiB, xr, lane4_of(lane), dB, eB);
        const float s0 = f16_lo(s[0]), s1 = f16_hi(s[0]), s2 = f16_lo(s[1]), s3 = f16_hi(s[1]);
#pragma unroll
        for (int pp = 0; pp < MP; ++pp) {
            const float d0 = use_a ? dA[pp][0] + eA[pp][0] : dB[pp][0] + eB[pp][0];
            const float d1 = use_a ? dA[pp][1] + eA[pp][1] : dB[pp][1] + eB[pp][1];
            const float d2 = use_a ? dA[pp][2] + eA[pp][2] : dB[pp][2] + eB[pp][2];
            const float d3 = use_a ? dA[pp][3] + eA[pp][3] : dB[pp][3] + eB[pp][3];
            acc_lo[pp] = fmaf(s0, d0, acc_lo[pp]);
            acc_lo[pp] = fmaf(s1, d1, acc_lo[pp]);
            acc_hi[pp] = fmaf(s2, d2, acc_hi[pp]);
            acc_hi[pp] = fmaf(s3, d3, acc_hi[pp]);
        }
    };
    auto load_x = [&](uint32_t xa, uint32_t (&xr)[16]) {
        uint4 x0, x1, x2, x3;
        if (kXEmb) {
            x0 = lds128<0>(xa);
            x1 = lds128<256>(xa);
            x2 = lds128<512>(xa);
            x3 = lds128<768>(xa);
        } else {
            x0 = lds128<0>(xa);
            x1 = lds128<128>(xa);
            x2 = lds128<256>(xa);
            x3 = lds128<384>(xa);
        }
        const uint32_t v[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                                x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
#pragma unroll
        for (int i = 0; i < 16; ++i) xr[i] = v[i];
    };

    bool started = false;
    uint32_t xlane = 0;
    int slot = 0;
    uint32_t fparity = 0;
    for (int pt0 = 0; pt0 < T; pt0 += p.PT) {
        const int pt1 = min(T, pt0 + p.PT);
        if (!started) {
            asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
            // formed after the first consumer barrier: the empty asm keeps every
            // x read below it
            xlane = base + (kXEmb ? 128u : p.x_off) + ((g >> 1) & 1) * kXSpan + (g & 1) * 64 + tq * 16;
            asm volatile("" : "+r"(xlane)::"memory");
            started = true;
        }
        for (int t = pt0; t < pt1; ++t) {
            float acc_lo[MP], acc_hi[MP];
#pragma unroll
            for (int pp = 0; pp < MP; ++pp) acc_lo[pp] = acc_hi[pp] = 0.f;
            for (int c = 0; c < (kWhole ? 1 : p.C); ++c) {
                if (!bad && !mbar_wait(bars + 8u * slot, fparity)) {
                    bad = true;
                    if (lane == 0) atomicOr(&g_gemv_m1_error, 0x800u);
                }
                const int units = kWhole ? upk : (min(p.KC, p.rowbytes - c * p.KC) + 127) >> 7;
                const uint32_t a0 = ring_lane + slot * p.stage_bytes + 128 * warp;
#pragma unroll
                for (int j = 0; j < kUPW; ++j) {
                    if (!bad && warp + kCW * j < units) {
                        if (kWhole) {
                            unit(a0 + 128 * kCW * j, xw[j], sc[0][j], acc_lo, acc_hi);
                        } else {
                            uint32_t xr[MP][16];
                            load_x(xlane + static_cast<uint32_t>(c * upk + warp + kCW * j) * (2 * kXSpan),
                                   xr[0]);
                            unit(a0 + 128 * kCW * j, xr, sc[0][j], acc_lo, acc_hi);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + 8u * (NS + slot));
                if (++slot == NS) {
                    slot = 0;
                    fparity ^= 1u;
                }
#pragma unroll
                for (int i = 0; i < kAhead - 1; ++i)
#pragma unroll
                    for (int j = 0; j < kUPW; ++j) {
                        sc[i][j][0] = sc[i + 1][j][0];
                        sc[i][j][1] = sc[i + 1][j][1];
                    }
                next_scales(sc[kAhead - 1]);
            }
            // lanes tq = 0, 1 hold the two spans' sums of rows g, g + 8 for
            // token 2 pp; lanes tq = 2, 3 the same for token 2 pp + 1
#pragma unroll
            for (int pp = 0; pp < MP; ++pp) {
                acc_lo[pp] += __shfl_xor_sync(0xFFFFFFFFu, acc_lo[pp], 1);
                acc_hi[pp] += __shfl_xor_sync(0xFFFFFFFFu, acc_hi[pp], 1);
                const int tok = 2 * pp + (tq >> 1);
                if ((tq & 1) == 0 && tok < MT) {
                    // this warp's partials of the tile's rows:
                    // slot [tile][warp][token][row]
                    float* slot_w = acc_s + (((t - pt0) * kCW + warp) * MT + tok) * 16;
                    slot_w[g] = acc_lo[pp];
                    slot_w[g + 8] = acc_hi[pp];
                }
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
        const int row_end = min(nrows, 16 * pt1);
        for (int r = 16 * pt0 + tid; r < row_end; r += kCW * 32) {
            const int rl = r - 16 * pt0;
#pragma unroll
            for (int tok = 0; tok < MT; ++tok) {
                if (tok >= p.M) break;
                const float* q = acc_s + ((rl >> 4) * kCW * MT + tok) * 16 + (rl & 15);
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < kCW; ++w) sum += q[16 * MT * w];
                if (Q4_IN_BOUNDS(static_cast<int64_t>(tok) * p.N + r0 + r, 1, static_cast<int64_t>(p.M) * p.N))
                    p.y[static_cast<int64_t>(tok) * p.N + r0 + r] = sum;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
    }
}

template <bool kEvenG, bool kWhole, bool kXEmb, int MT = 1>
cudaError_t launch_variant(const M1& p, int grid, int smem, int slot, cudaStream_t s,
                           const DeviceInfo& dev) {
    auto kern = gemv_m1_kernel<kEvenG, kWhole, kXEmb, MT>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem, slot, dev.device);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

// ---------------------------------------------------------------------------
// q4_wait_selftest: the bounded wait above, made to run out on purpose with
// nothing in flight (no copy, no tensor-memory allocation): one thread waits
// on an mbarrier that expects one arrival and gets it only if `arrive`.
// ---------------------------------------------------------------------------
__device__ unsigned long long g_selftest_waited_ns;

__global__ void wait_selftest_kernel(unsigned long long limit_ns, int arrive) {
    __shared__ __align__(8) unsigned long long bar_storage;
    if (threadIdx.x != 0) return;
    const uint32_t bar = smem_u32(&bar_storage);
    mbar_init(bar, 1);
    fence_mbar_init();
    if (arrive) mbar_arrive(bar);
    const unsigned long long t0 = globaltimer_ns();
    const bool ok = mbar_wait(bar, 0u, limit_ns);
    g_selftest_waited_ns = globaltimer_ns() - t0;
    if (!ok) atomicOr(&g_gemv_m1_error, 0x80u);
}

cudaError_t run_wait_selftest(uint32_t limit_us, int arrive, uint32_t* waited_us) {
    wait_selftest_kernel<<<1, 32>>>(static_cast<unsigned long long>(limit_us) * 1000ull, arrive);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    unsigned long long ns = 0;
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&ns, g_selftest_waited_ns, sizeof(ns));
    if (e == cudaSuccess) *waited_us = static_cast<uint32_t>(ns / 1000ull);
    return e;
}

cudaError_t take_gemv_m1_error(unsigned int* out) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_gemv_m1_error, sizeof(unsigned int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_gemv_m1_error, &zero, sizeof(unsigned int));
    return e;
}

cudaError_t launch_gemv_m1(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                           const uint16_t* x, float* y, int M, int64_t N, int64_t K, cudaStream_t s,
                           const DeviceInfo& dev) {
    if (dev.smem_reserved != kBase || M < 1 || M > 4) return cudaErrorNotSupported;
    M1 p{};
    p.M = M;
    p.codes = codes;
    p.scales = scales;
    p.cb = cb;
    p.x = x;
    p.y = y;
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.G = static_cast<int>(K / kGroup);
    p.S = (p.K + kSpan - 1) / kSpan;
    p.SP = p.S + (p.S & 1);
    p.rowbytes = p.K / 2;
    // A stage is 16 rows x KC bytes.  Rows up to 2 KB whose length is a
    // multiple of 128 bytes travel whole (a tile is one contiguous copy);
    // longer rows in C segments of KC bytes (a multiple of 128).
    const bool whole = p.rowbytes <= kMaxKC && p.rowbytes % 128 == 0;
    if (M > 1 && !whole) return cudaErrorNotSupported;  // several tokens: whole rows only
    const int mt = M == 1 ? 1 : (M == 2 ? 2 : 4);        // token slots
    if (whole) {
        p.C = 1;
        p.KC = p.rowbytes;
    } else {
        p.C = (p.rowbytes + kMaxKC - 1) / kMaxKC;
        p.KC = ((p.rowbytes + p.C - 1) / p.C + 127) / 128 * 128;
    }
    if (p.K > kXRounds * kCW * 32 * 8) return cudaErrorNotSupported;
    const bool xemb = p.SP <= kXEmbedSpans;
    p.stage_bytes = static_cast<uint32_t>(16 * p.KC);
    // Shared memory: table | row partials (PT tiles) | barriers | x (when not
    // in the table rows) | ring.  The ring's stage count is set with the
    // smallest partials area; the partials then take what the ring leaves,
    // up to kMaxPassTiles tiles (fewer passes, fewer barriers).
    auto layout = [&](int pt) {
        p.PT = pt;
        p.bar_off = kAccOff + static_cast<uint32_t>(pt * mt) * kTileSlotBytes;
        p.x_off = p.bar_off + 128u;
        const uint32_t x_end = xemb ? p.x_off : p.x_off + static_cast<uint32_t>(p.SP) * 512u;
        p.ring_off = (x_end + 127u) & ~127u;
        return dev.smem_optin - static_cast<int>(p.ring_off) - 128;  // 128: read slack
    };
    int ns = layout(kMinPassTiles) / static_cast<int>(p.stage_bytes);
    if (ns > kMaxStages) ns = kMaxStages;
    if (ns < 2) return cudaErrorNotSupported;
    p.NS = ns;
    const int64_t tiles_per_cta = ((N + dev.sm_count - 1) / dev.sm_count + 15) / 16 + 1;
    const int pt_cap = static_cast<int>(tiles_per_cta < kMaxPassTiles ? tiles_per_cta : kMaxPassTiles);
    for (int pt = pt_cap; pt > kMinPassTiles; --pt)
        if (layout(pt) >= ns * static_cast<int>(p.stage_bytes)) break;
    if (layout(p.PT) < ns * static_cast<int>(p.stage_bytes)) layout(kMinPassTiles);
    const int smem = static_cast<int>(p.ring_off + ns * p.stage_bytes) + 128;

    const int64_t tiles = (N + 15) / 16;
    const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
    const bool even = (p.G & 1) == 0;
    if (whole && mt == 2)
        return even ? launch_variant<true, true, true, 2>(p, grid, smem, 22, s, dev)
                    : launch_variant<false, true, true, 2>(p, grid, smem, 23, s, dev);
    if (whole && mt == 4)
        return even ? launch_variant<true, true, true, 4>(p, grid, smem, 24, s, dev)
                    : launch_variant<false, true, true, 4>(p, grid, smem, 25, s, dev);
    if (whole) {
        return even ? launch_variant<true, true, true>(p, grid, smem, 16, s, dev)
                    : launch_variant<false, true, true>(p, grid, smem, 17, s, dev);
    }
    if (xemb)
        return even ? launch_variant<true, false, true>(p, grid, smem, 18, s, dev)
                    : launch_variant<false, false, true>(p, grid, smem, 19, s, dev);
    return even ? launch_variant<true, false, false>(p, grid, smem, 20, s, dev)
                : launch_variant<false, false, false>(p, grid, smem, 21, s, dev);
}

Q4_DEFINE_TAKE_BOUNDS(gemv_m1)

}  // namespace q4
