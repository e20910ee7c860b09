// q4_api.cu -- the C ABI of q4.h: argument validation, the architecture
// gate, a per-device property cache, and dispatch to the kernel launchers.
#include <atomic>
#include <mutex>

#include "q4_internal.cuh"

namespace q4 {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxSlots = 96;

struct Cache {
    std::mutex mu;
    bool valid[kMaxDevices] = {};
    DeviceInfo info[kMaxDevices];
    std::atomic<int> smem_done[kMaxDevices][kMaxSlots];
    Cache() {
        for (auto& row : smem_done)
            for (auto& v : row) v.store(0, std::memory_order_relaxed);
    }
};

Cache& cache() {
    static Cache c;
    return c;
}

thread_local int g_last_cuda_error = 0;

q4_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = static_cast<int>(e);
    return Q4_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

q4_status check_K(int64_t K) {
    if (K <= 0 || K % kGroup != 0 || K > Q4_MAX_K) return Q4_ERR_SHAPE;
    return Q4_OK;
}

// Architecture gate plus property lookup for the current device.
q4_status gate(DeviceInfo* dev) {
    cudaError_t e = current_device_info(dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev->cc_major != 10 || dev->cc_minor != 0) return Q4_ERR_ARCH;
    return Q4_OK;
}

q4_status after_launch(cudaError_t e) {
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return Q4_OK;
}

q4_status check_matmul(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                       const uint16_t* x, float* y, int64_t M, int64_t N, int64_t K,
                       bool* empty) {
    *empty = false;
    q4_status st = check_K(K);
    if (st != Q4_OK) return st;
    if (M < 0 || N < 0 || M > Q4_MAX_MN || N > Q4_MAX_MN) return Q4_ERR_SHAPE;
    if (M == 0 || N == 0) {
        *empty = true;
        return Q4_OK;
    }
    if (!codes || !scales || !cb || !x || !y) return Q4_ERR_NULL;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(cb) || !aligned16(x) ||
        !aligned16(y))
        return Q4_ERR_ALIGN;
    return Q4_OK;
}

// q4_gemm's kernel choice, after validation.
q4_status gemm_dispatch(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb,
                        const uint16_t* x, float* y, int64_t M, int64_t N, int64_t K,
                        cudaStream_t stream, const DeviceInfo& dev) {
    if (M <= 16)
        return after_launch(launch_small_m(codes, scales, cb, x, y, static_cast<int>(M), N, K, stream, dev));
    if (M <= 24) {
        // still weight-streaming: the CUDA-core decode kernel beats the
        // tensor-core pipeline up to 24 tokens (measured crossover on B200)
        cudaError_t e = launch_gemm_small(codes, scales, cb, x, y, static_cast<int>(M), N, K, stream, dev);
        if (e != cudaErrorNotSupported) return after_launch(e);
        (void)cudaGetLastError();
    }
    return after_launch(launch_prefill(codes, scales, cb, x, y, M, N, K, stream, dev));
}

}  // namespace

cudaError_t current_device_info(DeviceInfo* info) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    Cache& c = cache();
    std::lock_guard<std::mutex> lock(c.mu);
    if (!c.valid[dev]) {
        DeviceInfo d{};
        d.device = dev;
        if ((e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) ||
            (e = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) ||
            (e = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) ||
            (e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                        dev)) ||
            (e = cudaDeviceGetAttribute(&d.smem_reserved, cudaDevAttrReservedSharedMemoryPerBlock,
                                        dev)))
            return e;
        c.info[dev] = d;
        c.valid[dev] = true;
    }
    *info = c.info[dev];
    return cudaSuccess;
}

cudaError_t ensure_smem_attr(const void* func, int bytes, int slot, int device) {
    if (slot < 0 || slot >= kMaxSlots || device < 0 || device >= kMaxDevices)
        return cudaErrorInvalidValue;
    std::atomic<int>& done = cache().smem_done[device][slot];
    if (done.load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) {
        int prev = done.load(std::memory_order_relaxed);
        while (prev < bytes && !done.compare_exchange_weak(prev, bytes)) {
        }
    }
    return e;
}

}  // namespace q4

using namespace q4;

// Two device slots fed from host memory (see q4_ring_create in q4.h).
struct q4_ring {
    std::mutex mu;
    int device = 0;
    int64_t slot_bytes = 0;
    void* slot[2] = {nullptr, nullptr};
    cudaStream_t copy = nullptr;
    cudaEvent_t copied[2] = {nullptr, nullptr};  // slot s holds the weights of its latest call
    cudaEvent_t used[2] = {nullptr, nullptr};    // the matmul that last read slot s is done
    int next = 0;
};

// A recorded decode step (see q4_step_create in q4.h).
struct q4_step {
    int device = 0;
    cudaStream_t capture = nullptr;
    cudaGraphExec_t exec = nullptr;
};

extern "C" {

q4_status q4_pack(const float* w, const uint16_t* codebook, uint8_t* codes, uint16_t* scales,
                  int64_t N, int64_t K, q4_stream_t stream) {
    q4_status st = check_K(K);
    if (st != Q4_OK) return st;
    if (N < 0 || N > Q4_MAX_MN) return Q4_ERR_SHAPE;
    if (N == 0) return Q4_OK;
    if (!w || !codebook || !codes || !scales) return Q4_ERR_NULL;
    if (!aligned16(w) || !aligned16(codebook) || !aligned16(codes) || !aligned16(scales))
        return Q4_ERR_ALIGN;
    DeviceInfo dev;
    if ((st = gate(&dev)) != Q4_OK) return st;
    return after_launch(launch_pack(w, codebook, codes, scales, N, K, stream, dev));
}

q4_status q4_dequant(const uint8_t* codes, const uint16_t* scales, const uint16_t* codebook,
                     float* w_out, int64_t N, int64_t K, q4_stream_t stream) {
    q4_status st = check_K(K);
    if (st != Q4_OK) return st;
    if (N < 0 || N > Q4_MAX_MN) return Q4_ERR_SHAPE;
    if (N == 0) return Q4_OK;
    if (!codes || !scales || !codebook || !w_out) return Q4_ERR_NULL;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(codebook) || !aligned16(w_out))
        return Q4_ERR_ALIGN;
    DeviceInfo dev;
    if ((st = gate(&dev)) != Q4_OK) return st;
    return after_launch(launch_dequant(codes, scales, codebook, w_out, N, K, stream, dev));
}

q4_status q4_embed_rows(const uint8_t* codes, const uint16_t* scales, const uint16_t* codebook,
                        const int32_t* ids, float* out, int64_t n_ids, int64_t N, int64_t K,
                        q4_stream_t stream) {
    q4_status st = check_K(K);
    if (st != Q4_OK) return st;
    if (N < 0 || N > Q4_MAX_MN || n_ids < 0 || n_ids > Q4_MAX_MN) return Q4_ERR_SHAPE;
    if (n_ids == 0) return Q4_OK;
    if (!codes || !scales || !codebook || !ids || !out) return Q4_ERR_NULL;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(codebook) || !aligned16(ids) ||
        !aligned16(out))
        return Q4_ERR_ALIGN;
    DeviceInfo dev;
    if ((st = gate(&dev)) != Q4_OK) return st;
    return after_launch(launch_embed_rows(codes, scales, codebook, ids, out, n_ids, N, K, stream, dev));
}

q4_status q4_gemv(const uint8_t* codes, const uint16_t* scales, const uint16_t* codebook,
                  const uint16_t* x, float* y, int64_t M, int64_t N, int64_t K,
                  q4_stream_t stream) {
    if (M != 1) return Q4_ERR_SHAPE;
    bool empty;
    q4_status st = check_matmul(codes, scales, codebook, x, y, M, N, K, &empty);
    if (st != Q4_OK || empty) return st;
    DeviceInfo dev;
    if ((st = gate(&dev)) != Q4_OK) return st;
    return after_launch(launch_small_m(codes, scales, codebook, x, y, 1, N, K, stream, dev));
}

q4_status q4_gemm(const uint8_t* codes, const uint16_t* scales, const uint16_t* codebook,
                  const uint16_t* x, float* y, int64_t M, int64_t N, int64_t K,
                  q4_stream_t stream) {
    bool empty;
    q4_status st = check_matmul(codes, scales, codebook, x, y, M, N, K, &empty);
    if (st != Q4_OK || empty) return st;
    DeviceInfo dev;
    if ((st = gate(&dev)) != Q4_OK) return st;
    return gemm_dispatch(codes, scales, codebook, x, y, M, N, K, stream, dev);
}

q4_status q4_gemm_noalloc(const uint8_t* codes, const uint16_t* scales, const uint16_t* codebook,
                          const uint16_t* x, float* y, int64_t M, int64_t N, int64_t K,
                          q4_stream_t stream) {
    bool empty;
    q4_status st = check_matmul(codes, scales, codebook, x, y, M, N, K, &empty);
    if (st != Q4_OK || empty) return st;
    if (M > 16 && static_cast<uint64_t>(M) * static_cast<uint64_t>(K) * sizeof(uint16_t) >
                      Q4_NOALLOC_SCRATCH_BYTES)
        return Q4_ERR_TOO_LARGE;
    DeviceInfo dev;
    if ((st = gate(&dev)) != Q4_OK) return st;
    if (M <= 16)
        return after_launch(
            launch_small_m(codes, scales, codebook, x, y, static_cast<int>(M), N, K, stream, dev));
    if (M <= 24) {
        cudaError_t e = launch_gemm_small(codes, scales, codebook, x, y, static_cast<int>(M), N, K,
                                          stream, dev);
        if (e != cudaErrorNotSupported) return after_launch(e);
        (void)cudaGetLastError();
    }
    return after_launch(launch_prefill_noalloc(codes, scales, codebook, x, y, M, N, K, stream, dev));
}

// Offset of the scales in a slot: after the codes, rounded up to 256 bytes.
static int64_t ring_scales_offset(int64_t N, int64_t K) { return (N * (K / 2) + 255) / 256 * 256; }

static void ring_free(q4_ring* r) {
    for (int s = 0; s < 2; ++s) {
        if (r->slot[s]) cudaFree(r->slot[s]);
        if (r->copied[s]) cudaEventDestroy(r->copied[s]);
        if (r->used[s]) cudaEventDestroy(r->used[s]);
    }
    if (r->copy) cudaStreamDestroy(r->copy);
    delete r;
}

q4_status q4_ring_create(int64_t slot_bytes, q4_ring** ring) {
    if (!ring) return Q4_ERR_NULL;
    *ring = nullptr;
    if (slot_bytes <= 0) return Q4_ERR_SHAPE;
    DeviceInfo dev;
    q4_status st = gate(&dev);
    if (st != Q4_OK) return st;
    q4_ring* r = new q4_ring();
    r->device = dev.device;
    r->slot_bytes = slot_bytes;
    cudaError_t e = cudaSuccess;
    for (int s = 0; s < 2 && e == cudaSuccess; ++s) {
        e = cudaMalloc(&r->slot[s], static_cast<size_t>(slot_bytes));
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r->copied[s], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r->used[s], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&r->copy, cudaStreamNonBlocking);
    if (e != cudaSuccess) {
        ring_free(r);
        return cuda_fail(e);
    }
    *ring = r;
    return Q4_OK;
}

q4_status q4_ring_destroy(q4_ring* ring) {
    if (!ring) return Q4_ERR_NULL;
    int cur = -1;
    cudaError_t e = cudaGetDevice(&cur);
    bool switched = false;
    if (e == cudaSuccess && cur != ring->device) {
        e = cudaSetDevice(ring->device);
        switched = e == cudaSuccess;
    }
    // wait for the ring's copies and for the matmuls that read its slots
    if (e == cudaSuccess) e = cudaStreamSynchronize(ring->copy);
    for (int s = 0; s < 2 && e == cudaSuccess; ++s) e = cudaEventSynchronize(ring->used[s]);
    ring_free(ring);
    if (switched) cudaSetDevice(cur);
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

q4_status q4_ring_gemm(q4_ring* ring, const uint8_t* host_codes, const uint16_t* host_scales,
                       const uint16_t* codebook, const uint16_t* x, float* y, int64_t M, int64_t N,
                       int64_t K, q4_stream_t stream) {
    if (!ring) return Q4_ERR_NULL;
    bool empty;
    q4_status st = check_matmul(host_codes, host_scales, codebook, x, y, M, N, K, &empty);
    if (st != Q4_OK || empty) return st;
    const int64_t soff = ring_scales_offset(N, K);
    if (soff + N * (K / kGroup) * 2 > ring->slot_bytes) return Q4_ERR_TOO_LARGE;
    DeviceInfo dev;
    if ((st = gate(&dev)) != Q4_OK) return st;
    if (dev.device != ring->device) return cuda_fail(cudaErrorInvalidDevice);
    std::lock_guard<std::mutex> lock(ring->mu);
    const int s = ring->next;
    uint8_t* dcodes = static_cast<uint8_t*>(ring->slot[s]);
    uint16_t* dscales = reinterpret_cast<uint16_t*>(dcodes + soff);
    // the copy waits for the matmul that last read this slot
    cudaError_t e = cudaStreamWaitEvent(ring->copy, ring->used[s], 0);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(dcodes, host_codes, static_cast<size_t>(N * (K / 2)), cudaMemcpyHostToDevice,
                            ring->copy);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(dscales, host_scales, static_cast<size_t>(N * (K / kGroup) * 2),
                            cudaMemcpyHostToDevice, ring->copy);
    if (e == cudaSuccess) e = cudaEventRecord(ring->copied[s], ring->copy);
    // the matmul waits for the copy
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, ring->copied[s], 0);
    if (e != cudaSuccess) return cuda_fail(e);
    st = gemm_dispatch(dcodes, dscales, codebook, x, y, M, N, K, stream, dev);
    if (st != Q4_OK) return st;
    e = cudaEventRecord(ring->used[s], stream);
    if (e != cudaSuccess) return cuda_fail(e);
    ring->next = s ^ 1;
    return Q4_OK;
}

static void step_free(q4_step* st) {
    if (st->exec) cudaGraphExecDestroy(st->exec);
    if (st->capture) cudaStreamDestroy(st->capture);
    delete st;
}

q4_status q4_step_create(const q4_linear* linears, int64_t n, q4_step** step) {
    if (!step) return Q4_ERR_NULL;
    *step = nullptr;
    if (!linears) return Q4_ERR_NULL;
    if (n < 1) return Q4_ERR_SHAPE;
    for (int64_t i = 0; i < n; ++i) {
        const q4_linear& l = linears[i];
        bool empty;
        const q4_status st = check_matmul(l.codes, l.scales, l.codebook, l.x, l.y, l.M, l.N, l.K, &empty);
        if (st != Q4_OK) return st;
    }
    DeviceInfo dev;
    q4_status st = gate(&dev);
    if (st != Q4_OK) return st;
    for (int64_t i = 0; i < n; ++i)
        if (linears[i].M > 16 && linears[i].N > 0) {
            // the tensor-core path's fixed x array and event, set up outside the capture
            const cudaError_t e = prepare_prefill(dev);
            if (e != cudaSuccess) return cuda_fail(e);
            break;
        }
    q4_step* r = new q4_step();
    r->device = dev.device;
    cudaError_t e = cudaStreamCreateWithFlags(&r->capture, cudaStreamNonBlocking);
    // relaxed: the launchers may set a kernel's shared-memory attribute the
    // first time they see it, which is not a stream operation
    if (e == cudaSuccess) e = cudaStreamBeginCapture(r->capture, cudaStreamCaptureModeRelaxed);
    if (e != cudaSuccess) {
        step_free(r);
        return cuda_fail(e);
    }
    for (int64_t i = 0; i < n && st == Q4_OK; ++i) {
        const q4_linear& l = linears[i];
        if (l.M == 0 || l.N == 0) continue;
        st = gemm_dispatch(l.codes, l.scales, l.codebook, l.x, l.y, l.M, l.N, l.K, r->capture, dev);
    }
    cudaGraph_t graph = nullptr;
    e = cudaStreamEndCapture(r->capture, &graph);
    if (st == Q4_OK && e != cudaSuccess) st = cuda_fail(e);
    if (st == Q4_OK) {
        e = cudaGraphInstantiate(&r->exec, graph, 0);
        if (e != cudaSuccess) st = cuda_fail(e);
    }
    if (graph) cudaGraphDestroy(graph);
    if (st != Q4_OK) {
        step_free(r);
        return st;
    }
    *step = r;
    return Q4_OK;
}

q4_status q4_step_launch(q4_step* step, q4_stream_t stream) {
    if (!step) return Q4_ERR_NULL;
    const cudaError_t e = cudaGraphLaunch(step->exec, stream);
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

q4_status q4_step_destroy(q4_step* step) {
    if (!step) return Q4_ERR_NULL;
    step_free(step);
    return Q4_OK;
}

q4_status q4_wait_selftest(uint32_t limit_us, int arrive, uint32_t* waited_us) {
    if (!waited_us) return Q4_ERR_NULL;
    *waited_us = 0;
    if (limit_us < 1 || limit_us > 1000000u) return Q4_ERR_SHAPE;
    DeviceInfo dev;
    const q4_status st = gate(&dev);
    if (st != Q4_OK) return st;
    const cudaError_t e = run_wait_selftest(limit_us, arrive, waited_us);
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

q4_status q4_bounds_flags(uint32_t* flags) {
    if (!flags) return Q4_ERR_NULL;
    *flags = 0;
    cudaError_t e = cudaDeviceSynchronize();
    cudaError_t (*const take[6])(unsigned int*) = {take_bounds_gemv_m1, take_bounds_gemm_small,
                                                   take_bounds_gemm_tc, take_bounds_gemv,
                                                   take_bounds_pack, take_bounds_gemv2};
    for (int i = 0; i < 6 && e == cudaSuccess; ++i) {
        unsigned int v = 0;
        e = take[i](&v);
        if (v) *flags |= 1u << i;
    }
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_bounds_checked(void) {
#ifdef Q4_DEBUG
    return 1;
#else
    return 0;
#endif
}

const char* q4_status_string(q4_status status) {
    switch (status) {
        case Q4_OK: return "Q4_OK";
        case Q4_ERR_NULL: return "Q4_ERR_NULL: a required pointer is NULL";
        case Q4_ERR_SHAPE: return "Q4_ERR_SHAPE: bad M, N or K";
        case Q4_ERR_ALIGN: return "Q4_ERR_ALIGN: a pointer is not 16-byte aligned";
        case Q4_ERR_ARCH: return "Q4_ERR_ARCH: the current device is not sm_100";
        case Q4_ERR_CUDA: return "Q4_ERR_CUDA: a CUDA call or kernel launch failed";
        case Q4_ERR_TOO_LARGE:
            return "Q4_ERR_TOO_LARGE: 2 * M * K bytes exceed Q4_NOALLOC_SCRATCH_BYTES (q4_gemm_noalloc)";
    }
    return "unknown q4_status";
}

int q4_last_cuda_error(void) { return g_last_cuda_error; }

int q4_abi_version(void) { return Q4_ABI_VERSION; }

q4_status q4_pack2(const float* w, const uint16_t* codebook4, uint8_t* codes, uint16_t* scales,
                   int64_t N, int64_t K, q4_stream_t stream) {
    q4_status st = check_K(K);
    if (st != Q4_OK) return st;
    if (N < 0 || N > Q4_MAX_MN) return Q4_ERR_SHAPE;
    if (N == 0) return Q4_OK;
    if (!w || !codebook4 || !codes || !scales) return Q4_ERR_NULL;
    if (!aligned16(w) || !aligned16(codebook4) || !aligned16(codes) || !aligned16(scales))
        return Q4_ERR_ALIGN;
    DeviceInfo dev;
    if ((st = gate(&dev)) != Q4_OK) return st;
    return after_launch(launch_pack2(w, codebook4, codes, scales, N, K, stream, dev));
}

q4_status q4_dequant2(const uint8_t* codes, const uint16_t* scales, const uint16_t* codebook4,
                      float* w_out, int64_t N, int64_t K, q4_stream_t stream) {
    q4_status st = check_K(K);
    if (st != Q4_OK) return st;
    if (N < 0 || N > Q4_MAX_MN) return Q4_ERR_SHAPE;
    if (N == 0) return Q4_OK;
    if (!codes || !scales || !codebook4 || !w_out) return Q4_ERR_NULL;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(codebook4) || !aligned16(w_out))
        return Q4_ERR_ALIGN;
    DeviceInfo dev;
    if ((st = gate(&dev)) != Q4_OK) return st;
    return after_launch(launch_dequant2(codes, scales, codebook4, w_out, N, K, stream, dev));
}

q4_status q4_gemv2(const uint8_t* codes, const uint16_t* scales, const uint16_t* codebook4,
                   const uint16_t* x, float* y, int64_t N, int64_t K, q4_stream_t stream) {
    if (K > Q4_GEMV2_MAX_K) return Q4_ERR_SHAPE;
    bool empty;
    q4_status st = check_matmul(codes, scales, codebook4, x, y, 1, N, K, &empty);
    if (st != Q4_OK || empty) return st;
    DeviceInfo dev;
    if ((st = gate(&dev)) != Q4_OK) return st;
    cudaError_t e = launch_gemv2(codes, scales, codebook4, x, y, N, K, stream, dev);
    if (e == cudaErrorNotSupported) {
        (void)cudaGetLastError();
        return Q4_ERR_SHAPE;
    }
    return after_launch(e);
}

q4_status q4_timeout_flags(uint32_t* flags) {
    if (!flags) return Q4_ERR_NULL;
    *flags = 0;
    unsigned int a = 0, b = 0, c = 0, d = 0;
    cudaError_t e = take_gemv_m1_error(&a);
    if (e == cudaSuccess) e = take_gemm_tc_error(&b);
    if (e == cudaSuccess) e = take_gemm_small_error(&c);
    if (e == cudaSuccess) e = take_gemv2_error(&d);
    if (e != cudaSuccess) return cuda_fail(e);
    *flags = (a & 0x0FF0u) | (d & 0x000Eu) | ((c & 0x0F00u) << 4) | ((b & 0xFFFFu) << 16);
    return Q4_OK;
}

}  // extern "C"
