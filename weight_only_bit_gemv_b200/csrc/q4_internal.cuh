// q4_internal.cuh -- internal declarations and device helpers of the sm_100a
// 4-bit codebook linear-layer library.  Not part of the public ABI (q4.h).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "q4.h"

namespace q4 {

constexpr int kGroup = 64;  // weights per scale group, along K

// ---------------------------------------------------------------------------
// per-device properties, queried once per device (q4_api.cu)
// ---------------------------------------------------------------------------
struct DeviceInfo {
    int device;
    int sm_count;
    int cc_major, cc_minor;
    int smem_optin;  // max dynamic shared memory per block (opt-in)
    int smem_reserved;  // shared memory the system reserves per block (ahead of user shared memory)
};
// Fills *info for the current device; returns cudaSuccess or the failing code.
cudaError_t current_device_info(DeviceInfo* info);

// Calls cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per device and
// kernel; `slot` identifies the kernel (a small dense index per translation
// unit range, see the launchers).
cudaError_t ensure_smem_attr(const void* func, int bytes, int slot, int device);

// ---------------------------------------------------------------------------
// launchers (each validated by q4_api.cu before it is called)
// ---------------------------------------------------------------------------
cudaError_t launch_pack(const float* w, const uint16_t* cb, uint8_t* codes, uint16_t* scales,
                        int64_t N, int64_t K, cudaStream_t s, const DeviceInfo& dev);
cudaError_t launch_dequant(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                           float* w, int64_t N, int64_t K, cudaStream_t s, const DeviceInfo& dev);
cudaError_t launch_embed_rows(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                             const int32_t* ids, float* out, int64_t n_ids, int64_t N, int64_t K,
                             cudaStream_t s, const DeviceInfo& dev);
// M in [1, 16]: decoded codebook values on mma.sync, exact products, fp32 sums.
cudaError_t launch_small_m(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                           const uint16_t* x, float* y, int M, int64_t N, int64_t K,
                           cudaStream_t s, const DeviceInfo& dev);
// M = 1 (and M = 2..4 with rows of at most 2 KB): bulk-copy-fed decode GEMV,
// one row range per CTA, launched with programmatic dependent launch.
// Returns cudaErrorNotSupported when the shape does not fit it (K too large
// for its shared-memory layout, or M > 1 with longer rows).
cudaError_t launch_gemv_m1(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                           const uint16_t* x, float* y, int M, int64_t N, int64_t K, cudaStream_t s,
                           const DeviceInfo& dev);
// M in [2, 32]: TMA-fed row blocks, decoded weights on mma.sync with the
// tokens as B columns, exact products.  Returns cudaErrorNotSupported when the
// device's shared-memory layout or the shape does not fit it.
cudaError_t launch_gemm_small(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                              const uint16_t* x, float* y, int M, int64_t N, int64_t K,
                              cudaStream_t s, const DeviceInfo& dev);
// M > 24 (and M = 17..24 when launch_gemm_small declines the shape):
// tcgen05 tensor-core GEMM with TMEM accumulators; x is converted to
// binary16 into a fixed device array whose users are ordered by one event
// per device.
// prepare_prefill sets up that array's address and event on `dev` (current):
// call it before a stream capture that may record the first such GEMM.
cudaError_t prepare_prefill(const DeviceInfo& dev);
cudaError_t launch_prefill(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                           const uint16_t* x, float* y, int64_t M, int64_t N, int64_t K,
                           cudaStream_t s, const DeviceInfo& dev);

// Size of q4_gemm's fixed device array for the binary16 copy of x (32 MiB
// per GPU); larger inputs run in chunks of tokens.
constexpr size_t kGemmXBytes = 32u << 20;

// launch_prefill with the x scratch in a fixed device array (q4_gemm_noalloc); the
// caller has checked 2 * M * K <= Q4_NOALLOC_SCRATCH_BYTES.
cudaError_t launch_prefill_noalloc(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                                   const uint16_t* x, float* y, int64_t M, int64_t N, int64_t K,
                                   cudaStream_t s, const DeviceInfo& dev);

// The two-bit variant (q2_codebook.cu): codes [N][K/4], a 4-entry codebook.
cudaError_t launch_pack2(const float* w, const uint16_t* cb, uint8_t* codes, uint16_t* scales,
                         int64_t N, int64_t K, cudaStream_t s, const DeviceInfo& dev);
cudaError_t launch_dequant2(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                            float* w, int64_t N, int64_t K, cudaStream_t s, const DeviceInfo& dev);
// One token; zeroes y on the stream, then adds into it.  Returns
// cudaErrorNotSupported when the staged x (136 bytes per group) does not fit
// the device's shared memory.
cudaError_t launch_gemv2(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                         const uint16_t* x, float* y, int64_t N, int64_t K, cudaStream_t s,
                         const DeviceInfo& dev);

// q4_wait_selftest's kernel (q4_gemv_m1.cu): a bounded mbarrier wait of at
// most limit_us that runs out unless `arrive`; synchronizes the device.
cudaError_t run_wait_selftest(uint32_t limit_us, int arrive, uint32_t* waited_us);

// Copy out and clear the timeout bits that a kernel family's bounded waits
// set (synchronous; see q4_timeout_flags).
cudaError_t take_gemv_m1_error(unsigned int* out);
cudaError_t take_gemm_tc_error(unsigned int* out);
cudaError_t take_gemm_small_error(unsigned int* out);
cudaError_t take_gemv2_error(unsigned int* out);

// ---------------------------------------------------------------------------
// bounds checks of the debug build (-DQ4_DEBUG, built as libq4_debug.so)
// ---------------------------------------------------------------------------
// Q4_IN_BOUNDS(first, count, extent): the elements [first, first + count) of a
// buffer of `extent` elements all exist.  In the debug build a failed check
// sets this translation unit's bit in its own device word and the caller skips
// the access (a skipped bulk copy leaves its mbarrier short, so the waits
// behind it run out and report too); nothing traps.  In the release build the
// check is the constant true and costs nothing.
#ifdef Q4_DEBUG
static __device__ unsigned int g_bounds_error_tu;
__device__ __forceinline__ bool q4_in_bounds(long long first, long long count, long long extent) {
    const bool ok = first >= 0 && count >= 0 && first + count <= extent;
    if (!ok) atomicOr(&g_bounds_error_tu, 1u);
    return ok;
}
#define Q4_IN_BOUNDS(first, count, extent) \
    q4::q4_in_bounds(static_cast<long long>(first), static_cast<long long>(count), static_cast<long long>(extent))
// Copies out and clears this translation unit's word (defined once per .cu
// file by Q4_DEFINE_TAKE_BOUNDS).
#define Q4_DEFINE_TAKE_BOUNDS(name)                                                        \
    cudaError_t take_bounds_##name(unsigned int* out) {                                   \
        unsigned int zero = 0;                                                             \
        cudaError_t e = cudaMemcpyFromSymbol(out, g_bounds_error_tu, sizeof(unsigned int)); \
        if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_bounds_error_tu, &zero, sizeof(unsigned int)); \
        return e;                                                                          \
    }
#else
#define Q4_IN_BOUNDS(first, count, extent) true
#define Q4_DEFINE_TAKE_BOUNDS(name)                          \
    cudaError_t take_bounds_##name(unsigned int* out) {      \
        *out = 0;                                            \
        return cudaSuccess;                                  \
    }
#endif
cudaError_t take_bounds_gemv_m1(unsigned int* out);
cudaError_t take_bounds_gemm_small(unsigned int* out);
cudaError_t take_bounds_gemm_tc(unsigned int* out);
cudaError_t take_bounds_gemv(unsigned int* out);
cudaError_t take_bounds_pack(unsigned int* out);
cudaError_t take_bounds_gemv2(unsigned int* out);

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 lds_u128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// Streaming 8-byte global load (evict-first); a plain load the compiler can schedule.
__device__ __forceinline__ uint2 ldg_stream_u2(const void* p) {
    return __ldcs(reinterpret_cast<const uint2*>(p));
}

__device__ __forceinline__ uint16_t ldg_u16(const void* p) {
    return __ldg(reinterpret_cast<const unsigned short*>(p));
}

// Shared-memory loads as plain C++ accesses: ordered after any asm volatile
// with a memory clobber (the mbarrier waits), otherwise free to be scheduled.
template <typename T>
__device__ __forceinline__ T ld_smem(const uint8_t* smem, uint32_t off) {
    return *reinterpret_cast<const T*>(smem + off);
}

// bfloat16 bits -> binary32 (exact)
__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) {
    return __uint_as_float(b << 16);
}

// D = A * B + C, m16n8k16, A row-major f16, B column-major f16, fp32 accumulators.
// Not volatile: a pure function of its registers, so the compiler may
// schedule it among the loads that feed it.
__device__ __forceinline__ void mma_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1,
                                          const float c[4]) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1),
          "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

}  // namespace q4
