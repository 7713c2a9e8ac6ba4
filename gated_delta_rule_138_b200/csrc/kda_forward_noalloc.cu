// kda_forward_noalloc: the tensor-core KDA forward without any device
// allocation, for callers that cannot call cudaMalloc.
//
// kda_forward allocates one device word per GPU (its timeout status word) the
// first time it runs the tensor-core kernel there.  Some callers cannot allow
// that: an inference server or training loop that reserves nearly all device
// memory for its own pool up front, a latency-critical loop where cudaMalloc
// may synchronise the device, or a host program that is not allowed to grow
// device memory once it has started.  This entry point keeps its scratch in a
// fixed, file-scope device array instead, so a call only launches the kernel.
//
// The scratch: one status word per (sequence, head) CTA, at most
// KDA_NOALLOC_MAX_SEQ_HEADS words (64 KiB).  Every GPU that loads the library
// holds this array until the process exits.  Each CTA always writes its own
// word (0 = finished, 1 = a bounded wait gave up), so nothing has to be cleared
// before a call.  All calls on a device share the array and it keeps the last
// call's contents; two calls that overlap on the GPU race on it.  The caller
// learns of a timeout by reading the words back with kda_noalloc_status, which
// allocates nothing either (a copy into caller-provided or stack host memory).
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "kda_sm100.cuh"

#include "../../include/kda.h"
#include "kda_common.cuh"

namespace kda {
void set_last_error_text(const char* text);
cudaError_t launch_chunk_tc_cta_status(const void* q, const void* k, const void* v,
                                       const void* alpha, const void* beta, const float* S0,
                                       const int32_t* cu, int nseq, void* out, float* S_final,
                                       int64_t rows, int64_t T, int H, int* status,
                                       cudaStream_t stream);
}  // namespace kda

static __device__ __align__(256) int g_kda_noalloc_status[KDA_NOALLOC_MAX_SEQ_HEADS];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_addr[kMaxDevices] = {};

// Device address of the scratch array for the current device.  In host code
// the array's name is only a host-side stand-in, so the address is taken from
// the runtime once per device (with that device current) and cached.  The
// cache assumes the device context lives as long as the process: after a
// cudaDeviceReset the module is loaded afresh and the cached address is stale,
// so a program that resets a device must not call these entry points again.
cudaError_t scratch_address(int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_addr[dev] == nullptr) {
        int* p = nullptr;
        e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_kda_noalloc_status);
        if (e != cudaSuccess) return e;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

kda_status_t fail_cuda(cudaError_t e) {
    char msg[256];
    std::snprintf(msg, sizeof(msg), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    kda::set_last_error_text(msg);
    return KDA_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" kda_status_t kda_forward_noalloc(const void* q, const void* k, const void* v,
                                            const void* alpha, const void* beta, const float* S0,
                                            const int32_t* cu_seqlens, int32_t num_seqs,
                                            void* out, float* S_final, int32_t B, int64_t T,
                                            int32_t H, int32_t d_k, int32_t d_v, int32_t chunk,
                                            kda_dtype_t in_dtype, kda_dtype_t out_dtype,
                                            kda_stream_t stream) {
    if (B < 0 || T < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if ((in_dtype != KDA_F32 && in_dtype != KDA_BF16) || (out_dtype != KDA_F32 && out_dtype != KDA_BF16))
        return KDA_ERR_INVALID_ARG;
    if (cu_seqlens != nullptr && (B != 1 || num_seqs < 0)) return KDA_ERR_INVALID_ARG;
    const int64_t nseq = cu_seqlens ? (int64_t)num_seqs : (int64_t)B;
    if ((int64_t)B * T > 0 && (!q || !k || !v || !alpha || !beta || !out))
        return KDA_ERR_INVALID_ARG;
    const void* p16[] = {q, k, v, alpha, S0, out, S_final};
    for (const void* p : p16)
        if (p && !aligned(p, 16)) return KDA_ERR_INVALID_ARG;
    if (!aligned(beta, 2) || !aligned(cu_seqlens, 4)) return KDA_ERR_INVALID_ARG;
    if (in_dtype != KDA_BF16 || out_dtype != KDA_BF16 || d_k != 128 || d_v != 128 || chunk != 64) {
        kda::set_last_error_text("kda_forward_noalloc: only bf16 in/out, d_k = d_v = 128, chunk 64");
        return KDA_ERR_UNSUPPORTED;
    }
    if (nseq * H > KDA_NOALLOC_MAX_SEQ_HEADS) {
        char msg[256];
        std::snprintf(msg, sizeof(msg),
                      "kda_forward_noalloc: %lld (sequence, head) pairs exceed the fixed scratch "
                      "of %d", (long long)(nseq * H), KDA_NOALLOC_MAX_SEQ_HEADS);
        kda::set_last_error_text(msg);
        return KDA_ERR_UNSUPPORTED;
    }
    const int64_t rows = cu_seqlens ? T : (int64_t)B * T;
    if (rows > 0x7fffffffLL || nseq > 65535 || H > 65535) return KDA_ERR_UNSUPPORTED;
    if (nseq == 0) return KDA_OK;
    kda::set_last_error_text("");
    int* status = nullptr;
    cudaError_t e = scratch_address(&status);
    if (e != cudaSuccess) return fail_cuda(e);
    e = kda::launch_chunk_tc_cta_status(q, k, v, alpha, beta, S0, cu_seqlens, (int)nseq, out,
                                        S_final, rows, T, H, status,
                                        reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e);
    // KDA_DEBUG set: wait for the call and report its status words, as kda_forward does
    // with its device status word
    const char* dbg = std::getenv("KDA_DEBUG");
    if (dbg && dbg[0] && dbg[0] != '0') return kda_noalloc_status((int32_t)(nseq * H), nullptr, stream);
    return KDA_OK;
}

namespace {
// Waits, bounded by limit_ns, on an mbarrier that nothing arrives on, then
// records the outcome in word `word` of the fixed array exactly as a forward
// CTA whose wait gave up does (1).  No fault, no hang.
__global__ void kda_noalloc_selftest_kernel(uint64_t limit_ns, int word) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        kda::sm100::mbar_init(&bar, 1);
        kda::sm100::mbar_fence_init();
    }
    __syncthreads();
    const bool done = kda::sm100::mbar_wait_ns(&bar, 0, limit_ns);
    if (threadIdx.x == 0) g_kda_noalloc_status[word] = done ? 0 : 1;
}
}  // namespace

extern "C" kda_status_t kda_noalloc_status(int32_t num_words, int32_t* host_words,
                                           kda_stream_t stream) {
    if (num_words < 0 || num_words > KDA_NOALLOC_MAX_SEQ_HEADS) return KDA_ERR_INVALID_ARG;
    int* unused = nullptr;
    cudaError_t e = scratch_address(&unused);   // loads the module on this device if needed
    if (e != cudaSuccess) return fail_cuda(e);
    e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e);
    bool any = false;
    constexpr int kBlock = 1024;
    int32_t buf[kBlock];
    for (int32_t w0 = 0; w0 < num_words; w0 += kBlock) {
        const int32_t n = num_words - w0 < kBlock ? num_words - w0 : kBlock;
        int32_t* dst = host_words ? host_words + w0 : buf;
        e = cudaMemcpyFromSymbol(dst, g_kda_noalloc_status, sizeof(int32_t) * (size_t)n,
                                 sizeof(int32_t) * (size_t)w0, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return fail_cuda(e);
        for (int32_t i = 0; i < n; ++i) any |= dst[i] != 0;
    }
    return any ? KDA_ERR_DEVICE_TIMEOUT : KDA_OK;
}

extern "C" kda_status_t kda_noalloc_selftest_timeout(uint64_t limit_ns, int32_t word,
                                                     kda_stream_t stream) {
    if (limit_ns == 0 || limit_ns > 10000000000ull) return KDA_ERR_INVALID_ARG;
    if (word < 0 || word >= KDA_NOALLOC_MAX_SEQ_HEADS) return KDA_ERR_INVALID_ARG;
    int* unused = nullptr;
    cudaError_t e = scratch_address(&unused);
    if (e != cudaSuccess) return fail_cuda(e);
    kda_noalloc_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns, word);
    e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : fail_cuda(e);
}
