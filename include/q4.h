/*
 * q4.h -- C ABI of the weight-only 4-bit codebook linear layer for NVIDIA
 * B200 (sm_100a), with a two-bit variant (q4_pack2, q4_dequant2, q4_gemv2).
 *
 * The operation.  A linear layer y = x * W^T whose weight matrix W [N][K]
 * (N outputs, K inputs) is stored as 4-bit codes into a 16-entry binary16
 * codebook, with one binary16 scale per group of 64 consecutive k of a row:
 *
 *     W[n][k] = codebook[code(n, k)] * scale[n][k / 64]
 *
 * This is the layout the "deep-fold" page describes in its "Method" section
 * (each group of 64 weights stores four-bit NF4 codes and one FP16 scale;
 * the packed payload is about 3.76x smaller than BF16).  The matmul entry
 * points rebuild W inside the kernel while they multiply, decoding each
 * weight from the codebook as it is used ("Trapetum" overview, "What it
 * does"), and never write a dense W to memory ("Trapetum" landing page, opening
 * paragraph; "deep-fold", "Method").  Decode (one token) is a GEMV and
 * prompt processing a tensor-core GEMM ("deep-fold", "Method" table).
 *
 * Layouts (all row-major and contiguous; there are no stride arguments):
 *   codes    uint8_t  [N][K/2]   byte j of row n holds code(n, 2j) in its low
 *                                nibble and code(n, 2j+1) in its high nibble
 *   scales   uint16_t [N][K/64]  binary16 bit patterns
 *   codebook uint16_t [16]       binary16 bit patterns (any values, any order)
 *   x        uint16_t [M][K]     bfloat16 bit patterns (M tokens)
 *   y        float    [M][N]     binary32, fully overwritten
 *   w        float    [N][K]     binary32 (input of q4_pack, output of q4_dequant)
 *
 * Ownership.  Every pointer is device memory owned by the caller (PyTorch,
 * cudaMalloc, ...), except the host-side weights of q4_ring_gemm.  The
 * library keeps no pointer after a call returns and holds only a per-device
 * cache of the device's properties.  The matmul, pack and dequant calls
 * allocate nothing at run time.  Two fixed device arrays are part of the
 * library's image, held by every GPU that loads it until the process exits:
 * 32 MiB for q4_gemm's binary16 copy of x (see q4_gemm) and 8 MiB for
 * q4_gemm_noalloc.  The library creates one event per device the first time
 * q4_gemm takes its tensor-core path there.  Explicitly created objects
 * allocate what their create call says: the two device slots of a q4_ring,
 * and the stream and graph of a q4_step.
 * All calls are asynchronous on the caller's stream (0 = legacy default
 * stream); none synchronizes the host except q4_timeout_flags and
 * q4_ring_destroy.  Inputs and outputs must not overlap.  The calls are
 * thread-safe.
 *
 * Errors.  Each call validates its arguments before launching anything, in
 * this order, and returns the first failure:
 *   Q4_ERR_SHAPE  K <= 0, K not a multiple of 64, K > Q4_MAX_K, M < 0, N < 0,
 *                 M or N above Q4_MAX_MN, or (q4_gemv only) M != 1
 *   (M == 0 or N == 0 is valid: Q4_OK is returned and nothing is launched)
 *   Q4_ERR_NULL   a required pointer is NULL
 *   Q4_ERR_ALIGN  a pointer is not 16-byte aligned
 *   Q4_ERR_ARCH   the current device is not compute capability 10.0 (sm_100)
 *   Q4_ERR_CUDA   a CUDA runtime call or the kernel launch failed; the CUDA
 *                 error code is available from q4_last_cuda_error()
 * Faults that happen while a kernel runs surface, as with any CUDA kernel, at
 * the caller's next synchronization.
 *
 * Input domain.  w finite with |w| <= 65504; x finite with |x| <= 65504; a
 * finite codebook.  Outside it results are unspecified.
 */
#ifndef Q4_H
#define Q4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (a CUstream_st pointer); pass a cudaStream_t. */
typedef struct CUstream_st* q4_stream_t;

typedef enum {
    Q4_OK = 0,
    Q4_ERR_NULL = 1,
    Q4_ERR_SHAPE = 2,
    Q4_ERR_ALIGN = 3,
    Q4_ERR_ARCH = 4,
    Q4_ERR_CUDA = 5,
    Q4_ERR_TOO_LARGE = 6  /* q4_gemm_noalloc only: x does not fit its fixed scratch */
} q4_status;

#define Q4_ABI_VERSION 1
#define Q4_GROUP 64
#define Q4_MAX_K (1 << 20)
#define Q4_MAX_MN 2147483647LL
/* Size of the fixed device scratch of q4_gemm_noalloc: 8 MiB per GPU. */
#define Q4_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * q4_pack -- quantize a dense binary32 W [N][K] into codes and scales.
 * Source: "deep-fold", "Method" (64-weight groups, four-bit codes, one FP16
 * scale; a CPU compressor writes them).  Per group of 64:
 *   scale = binary16(max |w|), rounded to nearest-even;
 *   code  = argmin_i |w / scale - codebook[i]|, the division and distances in
 *           binary32 (IEEE, round to nearest-even), ties to the lowest i;
 *   a scale that rounds to 0 gives every weight the index of the codebook
 *   entry of smallest magnitude.
 * Results are bit-identical to a serial IEEE implementation of these steps.
 * In: w [N][K] fp32, codebook [16].  Out: codes [N][K/2], scales [N][K/64].
 */
q4_status q4_pack(const float* w, const uint16_t* codebook, uint8_t* codes,
                  uint16_t* scales, int64_t N, int64_t K, q4_stream_t stream);

/*
 * q4_dequant -- write the dense binary32 W [N][K] = codebook[code] * scale.
 * The product of two binary16 values is exact in binary32, so the output is
 * exact.  For checking and debugging: the matmul entry points never call it.
 * In: codes, scales, codebook.  Out: w_out [N][K] fp32.
 */
q4_status q4_dequant(const uint8_t* codes, const uint16_t* scales,
                     const uint16_t* codebook, float* w_out, int64_t N,
                     int64_t K, q4_stream_t stream);

/*
 * q4_embed_rows -- dequantize only the requested rows of a packed matrix
 * (an embedding table): out[i][k] = codebook[code(ids[i], k)] *
 * scale[ids[i]][k / 64] in binary32, exact, as q4_dequant.
 * Source: "deep-fold", introduction and Figure 1 (embeddings, PackedEmbed,
 * decode only the requested rows, on a path of their own).
 * ids[i] outside [0, N) writes a row of zeros (ids live in device memory, so
 * they are not checked on the host).  Rows may repeat.
 * In: codes [N][K/2], scales [N][K/64], codebook, ids [n_ids] int32.
 * Out: out [n_ids][K] fp32.
 * Validation: Q4_ERR_SHAPE for a bad K (as q4_dequant), N or n_ids outside
 * [0, Q4_MAX_MN]; n_ids == 0 returns Q4_OK without a launch; then
 * Q4_ERR_NULL, Q4_ERR_ALIGN (every pointer 16-byte aligned), Q4_ERR_ARCH,
 * Q4_ERR_CUDA.
 */
q4_status q4_embed_rows(const uint8_t* codes, const uint16_t* scales,
                        const uint16_t* codebook, const int32_t* ids, float* out,
                        int64_t n_ids, int64_t N, int64_t K, q4_stream_t stream);

/*
 * q4_gemv -- one-token decode: y[0][n] = sum_k W[n][k] * x[0][k], M must be 1.
 * Source: "deep-fold", "Method" table (decode: a CUDA-core NF4 GEMV that
 * rebuilds values while it multiplies); "Trapetum" overview, "The bandwidth
 * law" (decode speed is set by the bytes of weights read).
 * Each weight is rebuilt in registers as binary16 codebook[code]; products
 * with x are exact and accumulate in binary32; the group's scale multiplies
 * the group's binary32 partial sum.  The result matches the exact sum to
 * within 1e-4 * sum_k |W x| + 1e-6 per element.  Each element of y is
 * written once by one thread block (no split of K across blocks), so the
 * result does not depend on timing.
 * Launch: with programmatic dependent launch.  The kernel may start while the
 * preceding kernel on the stream is still running; before it waits for that
 * kernel it only prefetches its inputs into L2 (which cannot return stale
 * data), and it reads every input after the preceding kernel has completed.
 * It also lets the next kernel start early; that kernel must itself wait
 * before reading y (kernels launched without the attribute always do).
 * In: codes, scales, codebook, x [1][K] bf16.  Out: y [1][N] fp32.
 */
q4_status q4_gemv(const uint8_t* codes, const uint16_t* scales,
                  const uint16_t* codebook, const uint16_t* x, float* y,
                  int64_t M, int64_t N, int64_t K, q4_stream_t stream);

/*
 * q4_gemm -- M tokens at once: y[m][n] = sum_k W[n][k] * x[m][k], any M >= 0.
 * Source: "deep-fold", "Method" table (prompt processing: a tensor-core NF4
 * GEMM that rebuilds weights into fragments); "Trapetum" overview, "What it
 * does" (speculative decoding verifies a few drafted tokens at once).
 * M <= 24 (verify batches, short prefill chunks) rebuilds binary16 codebook
 * values once per weight for all M tokens (mma.sync, tokens as columns):
 * exact products with binary32 accumulation, each group's sum scaled in
 * binary32, as q4_gemv.  M > 24 (prefill chunks) runs a tcgen05
 * tensor-core kernel: each weight is rebuilt as binary16(codebook * scale),
 * x is rounded to binary16, and products accumulate in binary32 in tensor
 * memory.  Either way the result is within 1e-4 * sum_k |W x| + 1e-6 of the
 * exact sum per element (for the tensor-core path this holds statistically:
 * the binary16 rounding of W is a relative error of at most 2^-11 per term,
 * which sums to about 1/(0.32 sqrt(K)) of the bound per standard deviation:
 * 20 at K = 4096, 7 at K = 512, but at K = 128 a few outputs in a million
 * can exceed the bound).
 * The tensor-core path first converts x to binary16 into a fixed 32 MiB
 * device array (see Ownership), in chunks of tokens when 2 * M * K is
 * larger.  Calls that take this path are ordered through one event per
 * device, so calls on different streams or host threads never use the array
 * at the same time (they may serialize on the GPU); under stream capture the
 * ordering becomes external event nodes of the graph.  The first such call on
 * a device looks up the array's address and creates the event: make it
 * before any stream capture (q4_step_create does this itself).  The
 * tensor-core kernel runs one persistent block per SM; where a tile's K range
 * is shared between blocks, that tile's y is zeroed first (by the x
 * conversion or a memset on the stream) and the partial sums are added into
 * it atomically, so the summation order (and the last bits of y) may vary
 * between runs.
 * In: codes, scales, codebook, x [M][K] bf16.  Out: y [M][N] fp32.
 */
q4_status q4_gemm(const uint8_t* codes, const uint16_t* scales,
                  const uint16_t* codebook, const uint16_t* x, float* y,
                  int64_t M, int64_t N, int64_t K, q4_stream_t stream);

/*
 * q4_gemm_noalloc -- q4_gemm for callers that may not allocate device memory.
 * The paper has no counterpart; this entry point exists for deployment.
 *
 * Some callers cannot let a library allocate device memory: engines that
 * reserve all device memory at start-up for a fixed arena and a KV cache
 * leave no headroom for allocations that come later, and hosts that account
 * for every byte themselves forbid hidden allocations.  q4_gemm allocates
 * nothing either, but it orders the users of its fixed array through an
 * event it creates, and it splits large inputs into chunks.  This call runs
 * the same kernels without that event or chunking: it keeps the binary16
 * copy of x in its own static device array of Q4_NOALLOC_SCRATCH_BYTES
 * (8 MiB), which every GPU that loads the library holds until the process
 * exits.  Its y agrees with q4_gemm's within the tolerance of q4_gemm.  It
 * calls no cudaMalloc, cudaFree, pool or event routine.
 *
 * Limits and hazards:
 *   - M > 16 needs 2 * M * K <= Q4_NOALLOC_SCRATCH_BYTES (e.g. M = 512 at
 *     K = 8192); larger inputs return Q4_ERR_TOO_LARGE before anything runs
 *     (for M = 17..24 this keeps room for the tensor-core path, which runs
 *     when the M <= 24 kernel declines a shape).  M <= 16 uses no scratch
 *     and has no such limit.
 *   - The array is shared by every call on a device and is not cleared
 *     between calls (each call overwrites what it reads).  Calls whose work
 *     can overlap on the GPU -- different streams, or different host threads
 *     -- race on it and may return wrong results; serialize them.
 *   - The first call that runs the tensor-core path on a device looks up the
 *     array's device address (a CUDA runtime query, no allocation) with that
 *     device current; make a first call with M > 24 before any stream
 *     capture.
 * Validation order: Q4_ERR_SHAPE, Q4_ERR_NULL, Q4_ERR_ALIGN (as q4_gemm), then
 * Q4_ERR_TOO_LARGE, Q4_ERR_ARCH, Q4_ERR_CUDA.
 * In and out: as q4_gemm.
 */
q4_status q4_gemm_noalloc(const uint8_t* codes, const uint16_t* scales,
                          const uint16_t* codebook, const uint16_t* x, float* y,
                          int64_t M, int64_t N, int64_t K, q4_stream_t stream);

/*
 * CopyRing -- matmuls whose packed weights live in host memory.
 * Source: "deep-fold", "Method" table (models that exceed the GPU budget:
 * selected packed matrices stream from pinned host memory through two
 * reusable GPU slots) and Figure 1 (overflow adds pinned host storage and two
 * reusable device slots, then the same GEMM kernel).
 *
 * q4_ring_create -- on the current device, allocate two device slots of
 * slot_bytes each (cudaMalloc), a copy stream and four events.  A slot must
 * hold a matrix's codes, padded to 256 bytes, plus its scales:
 * ceil(N * K / 2 / 256) * 256 + N * K / 32 bytes.  Returns Q4_ERR_NULL for a
 * NULL ring, Q4_ERR_SHAPE for slot_bytes <= 0, Q4_ERR_ARCH, Q4_ERR_CUDA.
 *
 * q4_ring_gemm -- y = x W^T exactly as q4_gemm (q4_gemv's kernel for M = 1),
 * with codes [N][K/2] and scales [N][K/64] in host memory.  The call
 * enqueues, without blocking the host:
 *   1. on the ring's copy stream, once the matmul that last read the ring's
 *      next slot has finished, the copy of codes and scales into that slot;
 *   2. on `stream`, once that copy has landed, the matmul on the slot.
 * Consecutive calls alternate the slots, so the copy of one call overlaps the
 * matmul of the one before.  Use page-locked host memory (cudaHostAlloc or
 * cudaHostRegister); pageable memory is correct but does not overlap.  The
 * host buffers must stay unchanged until the call's copy has run
 * (synchronize `stream`).  Calls on one ring are serialized by a mutex; each
 * must be made with the ring's device current (else Q4_ERR_CUDA,
 * cudaErrorInvalidDevice).  Validation as q4_gemm (the host pointers must be
 * 16-byte aligned), plus Q4_ERR_NULL for a NULL ring and Q4_ERR_TOO_LARGE
 * for a matrix larger than a slot.  Not capturable in a CUDA graph (it
 * records events on a stream of its own).
 *
 * q4_ring_destroy -- wait for the ring's copies and the matmuls that read its
 * slots, then free it.
 */
typedef struct q4_ring q4_ring;
q4_status q4_ring_create(int64_t slot_bytes, q4_ring** ring);
q4_status q4_ring_gemm(q4_ring* ring, const uint8_t* host_codes,
                       const uint16_t* host_scales, const uint16_t* codebook,
                       const uint16_t* x, float* y, int64_t M, int64_t N,
                       int64_t K, q4_stream_t stream);
q4_status q4_ring_destroy(q4_ring* ring);

/* Human-readable name of a status code (static storage, never NULL). */
const char* q4_status_string(q4_status status);

/* The cudaError_t value behind the last Q4_ERR_CUDA returned on this thread
 * (0 if none). */
int q4_last_cuda_error(void);

/* Q4_ABI_VERSION of the library that was loaded. */
int q4_abi_version(void);

/*
 * The two-bit variant: the same groups of 64 weights and binary16 scales,
 * 2-bit codes into a 4-entry binary16 codebook.
 * Source: "Trapetum" overview, "In one sentence" and "Frontier models on your
 * own hardware" (a 70B model in 2 bits on one 24 GB card).  The pages print
 * no 2-bit layout; this one is the 4-bit layout with four codes per byte:
 *   codes     uint8_t  [N][K/4]   byte j of row n holds code(n, 4j + i) in
 *                                 bits 2i and 2i + 1 (i = 0..3)
 *   scales    uint16_t [N][K/64]  binary16 bit patterns
 *   codebook4 uint16_t [4]        binary16 bit patterns (any values, any order)
 *   W[n][k] = codebook4[code(n, k)] * scale[n][k / 64]
 *
 * q4_pack2 / q4_dequant2: q4_pack / q4_dequant with 4 entries (nearest entry
 * in binary32, ties to the lowest index; a zero scale gives the entry of
 * smallest magnitude); bit-identical to a serial IEEE implementation.
 * q4_gemv2: one token, y[n] = sum_k W[n][k] * x[k], x [K] bfloat16, y [N]
 * fp32.  Products are exact (x rounded to binary16, as q4_gemv), the sums
 * fp32.  Up to K = 57344 each element of y is written once by one thread
 * block (programmatic dependent launch, as q4_gemv), so the result does not
 * depend on timing; above that, y is zeroed on the stream and then
 * accumulated by several thread blocks, so the order of the fp32 additions
 * is not fixed from run to run.
 * Validation as q4_dequant / q4_gemv (M = 1 implied), plus Q4_ERR_SHAPE for
 * K > Q4_GEMV2_MAX_K (x is staged in shared memory).
 */
#define Q4_GEMV2_MAX_K 98304
q4_status q4_pack2(const float* w, const uint16_t* codebook4, uint8_t* codes,
                   uint16_t* scales, int64_t N, int64_t K, q4_stream_t stream);
q4_status q4_dequant2(const uint8_t* codes, const uint16_t* scales,
                      const uint16_t* codebook4, float* w_out, int64_t N,
                      int64_t K, q4_stream_t stream);
q4_status q4_gemv2(const uint8_t* codes, const uint16_t* scales,
                   const uint16_t* codebook4, const uint16_t* x, float* y,
                   int64_t N, int64_t K, q4_stream_t stream);

/*
 * Decode steps as one CUDA graph.
 * Source: "deep-fold", "Method" table (the decode runs a full greedy step as
 * one CUDA graph); "Trapetum" landing page (the 7B decode rate it reports
 * with CUDA graphs).  A decode step launches the same linears on the same
 * buffers token after token; recording those launches once and replaying
 * them removes the host's launch cost from every token.
 *
 * q4_linear -- one linear of a step: y = x W^T with the arguments of q4_gemm
 * (M = 1 runs q4_gemv's kernel).  The pointers are baked into the step: to
 * run the next token, write new values into the same x buffers and launch
 * the step again.
 *
 * q4_step_create -- validate every linear as q4_gemm does (the first failure
 * is returned, and nothing is recorded), then record their launches, in list
 * order, on a private stream of the current device into a CUDA graph and
 * instantiate it.  Nothing runs.  Consecutive launches keep programmatic
 * dependent launch, so a kernel's start overlaps the end of the one before.
 * Linears with M == 0 or N == 0 are skipped.  Creates a stream and a graph
 * (host-side objects and the driver's own graph resources); no device memory
 * is allocated for the linears' data.  Returns Q4_ERR_NULL for a NULL list
 * or step, Q4_ERR_SHAPE for n < 1, the linears' validation errors,
 * Q4_ERR_ARCH, Q4_ERR_CUDA.
 *
 * q4_step_launch -- replay the recorded launches on `stream` (asynchronous;
 * the step's device must be current).  Replays on different streams that
 * overlap race on the linears' y buffers.
 *
 * q4_step_destroy -- free the graph and the stream (waits for nothing: let
 * the step's launches finish first).
 */
typedef struct {
    const uint8_t* codes;
    const uint16_t* scales;
    const uint16_t* codebook;
    const uint16_t* x;
    float* y;
    int64_t M, N, K;
} q4_linear;
typedef struct q4_step q4_step;
q4_status q4_step_create(const q4_linear* linears, int64_t n, q4_step** step);
q4_status q4_step_launch(q4_step* step, q4_stream_t stream);
q4_status q4_step_destroy(q4_step* step);

/*
 * q4_wait_selftest -- exercise the bounded wait the kernels use, with
 * nothing in flight: one thread block initializes an mbarrier that expects
 * one arrival, arrives on it only if `arrive` is nonzero, and waits on it for
 * at most limit_us microseconds (1..1000000) of the GPU's global timer.  A
 * wait that runs out sets bit 7 of q4_timeout_flags, exactly as a kernel's
 * wait that runs out sets its own bit, and the block returns.  The call
 * synchronizes the current device and stores in *waited_us how long the wait
 * took.  Not an operation of the method: a check of the failure detection.
 * Returns Q4_ERR_NULL for a NULL waited_us, Q4_ERR_SHAPE for a limit outside
 * 1..1000000, Q4_ERR_ARCH, Q4_ERR_CUDA.
 */
q4_status q4_wait_selftest(uint32_t limit_us, int arrive, uint32_t* waited_us);

/*
 * Bounds-checked build.  Built with -DQ4_DEBUG (python -m
 * weight_only_bit_gemv_b200.build --debug, which writes libq4_debug.so), every
 * kernel checks the global index ranges it computes -- bulk-copy and load
 * sources, scale copies, x reads, y writes -- against the buffers' extents
 * before each access.  A range that falls outside sets a bit and the access
 * is skipped (nothing traps; a skipped bulk copy leaves its mbarrier short and
 * the waits behind it run out and report through q4_timeout_flags).  Not an
 * operation of the method: a substitute for a memory checker.
 *
 * q4_bounds_flags -- synchronize the current device, store in *flags the bits
 * set by failed checks since the last call and clear them: bit 0 the M <= 4
 * decode kernel, 1 the M = 2..24 kernel, 2 the tensor-core GEMM, 3 the
 * fallback small-M kernel, 4 pack / dequant / embedding rows, 5 the two-bit
 * kernels.  Always 0 in a release build.  Returns Q4_ERR_NULL for a NULL
 * flags, Q4_ERR_CUDA if a CUDA call fails.
 *
 * q4_bounds_checked -- 1 if this library was built with the checks, else 0.
 */
q4_status q4_bounds_flags(uint32_t* flags);
int q4_bounds_checked(void);

/*
 * q4_timeout_flags -- every wait inside the bulk-copy and tensor-core
 * kernels is bounded (about two seconds); a wait that runs out sets a bit in
 * a device word, the kernel drains what it has in flight, frees its tensor
 * memory and exits, leaving its output incomplete.  This call synchronizes the
 * current device, stores the bits set since the last call in *flags and
 * clears them: bits 1-3 the two-bit GEMV (producer, drain and consumer
 * waits), bits 4-11 the M = 1 GEMV (bit 7: q4_wait_selftest's wait ran out;
 * bit 8: its shared-memory layout did not match the device; bits 9-11:
 * producer, drain and consumer waits), bits
 * 12-15 the M = 2..24 kernel (the same four conditions), bits 16-31 the
 * tensor-core GEMM (M > 24); 0 = none.  Not an operation of the method; a
 * health check.
 * Returns Q4_ERR_NULL for a NULL flags, Q4_ERR_CUDA if a CUDA call fails.
 */
q4_status q4_timeout_flags(uint32_t* flags);

#ifdef __cplusplus
}
#endif

#endif /* Q4_H */
