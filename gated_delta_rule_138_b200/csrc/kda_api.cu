// C ABI of libkda.so (declared in include/kda.h): argument validation and
// dispatch to the kernels.  No entry point allocates on the caller's behalf
// beyond the library-owned workspace, synchronises the device, or throws.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/kda.h"
#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {
cudaError_t launch_chunk_simt(int in_bf16, int out_bf16, int chunk, const void* q, const void* k,
                              const void* v, const void* alpha, const void* beta, const float* S0,
                              const int32_t* cu, int nseq, void* out, float* S_final, int64_t T,
                              int H, int DK, int DV, cudaStream_t s, const int32_t* slots = nullptr,
                              int num_slots = 0);
cudaError_t launch_decode(int in_bf16, int out_bf16, const void* q, const void* k, const void* v,
                          const void* alpha, const void* beta, float* S, void* out, int64_t NH,
                          int DK, int DV, cudaStream_t s, const int32_t* slots, int num_slots,
                          int H, int T = 1, int fused = 0);
cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const void* alpha,
                            const void* beta, const float* S0, const int32_t* cu, int nseq,
                            void* out, float* S_final, int64_t rows, int64_t T, int H, int* status,
                            cudaStream_t stream, const int32_t* slots = nullptr, int num_slots = 0,
                            int fused = 0);
size_t chunk_tc_segmented_workspace_bytes(int64_t nseq, int64_t rows, int H, int nseg);
size_t backward_workspace_floats(bool packed, int64_t nseq, int64_t T, int H, int DK, int DV);
cudaError_t launch_backward(int in_bf16, const void* q, const void* k, const void* v,
                            const void* alpha, const void* beta, const float* S0, const void* dout,
                            const float* dSf, const int32_t* cu, int64_t nseq, int64_t T, int H,
                            int DK, int DV, float* dq, float* dk, float* dv, float* dalpha,
                            float* dbeta, float* dS0, float* workspace, cudaStream_t s);
size_t backward_tc_workspace_bytes(bool packed, int64_t nseq, int64_t T, int H);
bool backward_tc_supported(bool bf16, int64_t nseq, int64_t T, int H, int DK, int DV, bool packed);
cudaError_t launch_backward_tc(const void* q, const void* k, const void* v, const void* alpha,
                               const void* beta, const float* S0, const void* dout,
                               const float* dSf, const int32_t* cu, int64_t nseq, int64_t T, int H,
                               float* dq, float* dk, float* dv, float* dalpha, float* dbeta,
                               float* dS0, void* workspace, int* status, cudaStream_t s);
cudaError_t launch_segment_maps(const void* k, const void* v, const void* alpha, const void* beta,
                                const int32_t* cu, int nseq, float* maps, int64_t rows, int64_t T,
                                int H, int* status, cudaStream_t stream);
cudaError_t launch_apply_maps(const float* S0, const float* maps, int G, int nseq, int H, float* out,
                              cudaStream_t stream);
cudaError_t launch_chunk_tc_segmented(const void* q, const void* k, const void* v,
                                      const void* alpha, const void* beta, const float* S0,
                                      const int32_t* cu, int nseq, void* out, float* S_final,
                                      int64_t rows, int64_t T, int H, int nseg, void* workspace,
                                      int* status, cudaStream_t stream, int fused = 0);
}  // namespace kda

namespace {

thread_local char g_last_error[256] = "";
std::atomic<uint64_t> g_launches{0};

kda_status_t cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return KDA_OK;
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e),
                  cudaGetErrorString(e));
    return KDA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool is_dtype(kda_dtype_t d) { return d == KDA_F32 || d == KDA_BF16; }
bool head_dim_ok(int32_t d) { return d == 64 || d == 128; }

bool use_tc(int32_t d_k, int32_t d_v, int32_t chunk, kda_dtype_t in, kda_dtype_t out) {
    return in == KDA_BF16 && out == KDA_BF16 && d_k == 128 && d_v == 128 && chunk == 64;
}

// One device status word per GPU: kernels set it when a bounded wait gives up.
constexpr int kMaxDevices = 64;
std::mutex g_status_mu;
int* g_status[kMaxDevices] = {};

cudaError_t device_status_word(int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_status[dev]) {
        int* p = nullptr;
        e = cudaMalloc(&p, sizeof(int));
        if (e != cudaSuccess) return e;
        e = cudaMemset(p, 0, sizeof(int));
        if (e != cudaSuccess) { cudaFree(p); return e; }
        g_status[dev] = p;
    }
    *out = g_status[dev];
    return cudaSuccess;
}

// One stream-ordered memory pool per GPU for the split forward's workspace.  It
// keeps what it has reserved (no release threshold), so that repeated calls reuse
// the same device memory instead of mapping it anew after every synchronisation;
// kda_release_workspace hands it back.
cudaMemPool_t g_pool[kMaxDevices] = {};

cudaError_t workspace_pool(cudaMemPool_t* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_pool[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        e = cudaMemPoolCreate(&pool, &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = UINT64_MAX;
        e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) { cudaMemPoolDestroy(pool); return e; }
        g_pool[dev] = pool;
    }
    *out = g_pool[dev];
    return cudaSuccess;
}

// Time segments per sequence for the tensor-core forward.  One CTA runs one
// (sequence, head) segment on one SM and a segment costs in proportion to its
// chunks.  A split runs every segment in the dual mode (kSplitChunk of an unsplit
// chunk: the 256-wide state and both output parts) and then a pass over the
// outputs, o += Qg S_g, bound by memory: per (sequence, head) about kSplitPass of
// the unsplit CTA's time (its traffic, 3 x 256 bytes per token, against a chunk's
// time per token).  The cost, in units of the unsplit CTA's time, of g segments is
// kSplitChunk * waves(units g) / g + kSplitPass * units / SMs + a small charge per
// segment (the scan's chain, the launches), with waves = ceil(CTAs / SMs); g = 1
// costs waves(units).  Segments keep >= 16 chunks.
constexpr double kSplitChunk = 1.15;
constexpr double kSplitPass = 0.15;
int segments_for(int64_t nseq, int64_t tokens_per_seq, int64_t H, int sms) {
    const int64_t units = nseq * H;
    if (units <= 0 || sms <= 0) return 1;
    const int64_t chunks = (tokens_per_seq + 63) / 64;
    const auto waves = [&](int64_t ctas) { return (double)((ctas + sms - 1) / sms); };
    double best = waves(units);
    int best_g = 1;
    for (int g = 2; g <= 64 && chunks >= (int64_t)g * 16 && nseq * g <= 65535; ++g) {
        const double cost = kSplitChunk * waves(units * g) / g + kSplitPass * units / sms + 0.0002 * g;
        if (cost < best) {
            best = cost;
            best_g = g;
        }
    }
    return best_g;
}

int current_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;   // no device visible: assume a B200
    }
    return sms;
}

// Dense multi-token steps of at most this many tokens per sequence take the
// token-sequential kernel (state in registers) instead of the chunk kernels.
constexpr int64_t kMaxStepTokens = 16;

bool debug_sync() {
    const char* v = std::getenv("KDA_DEBUG");
    return v && v[0] && v[0] != '0';
}

// Waits, bounded by limit_ns, on an mbarrier that nothing ever arrives on, and
// records the timeout in the device status word exactly as the forward kernel
// does.  No fault, no hang: the wait gives up and the kernel returns.
__global__ void kda_selftest_wait_kernel(int* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        kda::sm100::mbar_init(&bar, 1);
        kda::sm100::mbar_fence_init();
    }
    __syncthreads();
    const bool done = kda::sm100::mbar_wait_ns(&bar, 0, limit_ns);
    if (!done && threadIdx.x == 0) atomicExch(status, 1);
}

}  // namespace

namespace kda {
// Shared with the other entry-point files of the library: the text returned by
// kda_last_error for this thread.
void set_last_error_text(const char* text) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s", text ? text : "");
}
}  // namespace kda

extern "C" {

const char* kda_status_string(kda_status_t status) {
    switch (status) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_DEVICE_TIMEOUT: return "KDA_ERR_DEVICE_TIMEOUT";
    }
    return "KDA_ERR_UNKNOWN";
}

const char* kda_last_error(void) { return g_last_error; }

uint64_t kda_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* kda_forward_kernel_name(int32_t d_k, int32_t d_v, int32_t chunk,
                                    kda_dtype_t in_dtype, kda_dtype_t out_dtype) {
    if (!is_dtype(in_dtype) || !is_dtype(out_dtype)) return nullptr;
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v)) return nullptr;
    if (chunk != 16 && chunk != 32 && chunk != 64) return nullptr;
    return use_tc(d_k, d_v, chunk, in_dtype, out_dtype) ? "chunk_tc_bf16" : "chunk_simt_f32";
}

kda_status_t kda_device_status(kda_stream_t stream) {
    int* word = nullptr;
    cudaError_t e = device_status_word(&word);
    if (e != cudaSuccess) return cuda_status(e);
    e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e);
    int v = 0;
    e = cudaMemcpy(&v, word, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    if (v != 0) {
        e = cudaMemset(word, 0, sizeof(int));
        if (e != cudaSuccess) return cuda_status(e);
        return KDA_ERR_DEVICE_TIMEOUT;
    }
    return KDA_OK;
}

size_t kda_forward_workspace_bytes(int32_t B, int64_t T, int32_t H, int32_t d_k, int32_t d_v,
                                   int32_t chunk) {
    size_t bytes = sizeof(int);  // the per-device status word, allocated once
    if (B > 0 && T > 0 && H > 0 && use_tc(d_k, d_v, chunk, KDA_BF16, KDA_BF16)) {
        const int nseg = segments_for(B, T, H, current_sms());
        bytes += kda::chunk_tc_segmented_workspace_bytes(B, (int64_t)B * T, H, nseg);
    }
    return bytes;
}

kda_status_t kda_release_workspace(void) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kMaxDevices) return KDA_OK;
    cudaMemPool_t pool = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_status_mu);
        pool = g_pool[dev];
    }
    return pool ? cuda_status(cudaMemPoolTrimTo(pool, 0)) : KDA_OK;
}

int32_t kda_forward_segments(int32_t num_seqs, int64_t tokens_per_seq, int32_t H, int32_t num_sms) {
    if (num_seqs <= 0 || tokens_per_seq <= 0 || H <= 0) return 1;
    return segments_for(num_seqs, tokens_per_seq, H, num_sms > 0 ? num_sms : current_sms());
}

kda_status_t kda_selftest_timeout(uint64_t limit_ns, kda_stream_t stream) {
    if (limit_ns == 0 || limit_ns > 10000000000ull) return KDA_ERR_INVALID_ARG;
    int* status = nullptr;
    cudaError_t e = device_status_word(&status);
    if (e != cudaSuccess) return cuda_status(e);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    kda_selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status, limit_ns);
    return cuda_status(cudaGetLastError());
}

}  // extern "C"

namespace {

// kda_forward and kda_forward_fused; `fused`: logits for alpha and beta, q and k
// unnormalised (tensor-core kernel only).
kda_status_t forward_impl(const void* q, const void* k, const void* v, const void* alpha,
                          const void* beta, const float* S0, const int32_t* cu_seqlens,
                          int32_t num_seqs, void* out, float* S_final, int32_t B, int64_t T,
                          int32_t H, int32_t d_k, int32_t d_v, int32_t chunk,
                          kda_dtype_t in_dtype, kda_dtype_t out_dtype, kda_stream_t stream,
                          int fused) {
    if (B < 0 || T < 0 || H <= 0 || !is_dtype(in_dtype) || !is_dtype(out_dtype))
        return KDA_ERR_INVALID_ARG;
    if (cu_seqlens != nullptr && (B != 1 || num_seqs < 0)) return KDA_ERR_INVALID_ARG;
    const int64_t nseq = cu_seqlens ? (int64_t)num_seqs : (int64_t)B;
    const bool has_tokens = (int64_t)B * T > 0;
    if (has_tokens && (!q || !k || !v || !alpha || !beta || !out)) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, alpha, S0, out, S_final};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(beta, in_dtype == KDA_BF16 ? 2 : 4) || !aligned_to(cu_seqlens, 4))
        return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v)) return KDA_ERR_UNSUPPORTED;
    if (chunk != 16 && chunk != 32 && chunk != 64) return KDA_ERR_UNSUPPORTED;
    if (nseq > 65535 || H > 65535) return KDA_ERR_UNSUPPORTED;  // grid y/z limits
    if (fused && !use_tc(d_k, d_v, chunk, in_dtype, out_dtype)) {
        std::snprintf(g_last_error, sizeof(g_last_error),
                      "kda_forward_fused: only bf16 in/out, d_k = d_v = 128, chunk 64");
        return KDA_ERR_UNSUPPORTED;
    }
    if (nseq == 0) return KDA_OK;
    g_last_error[0] = '\0';
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int in_bf16 = in_dtype == KDA_BF16, out_bf16 = out_dtype == KDA_BF16;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (use_tc(d_k, d_v, chunk, in_dtype, out_dtype)) {
        int* status = nullptr;
        cudaError_t e = device_status_word(&status);
        if (e != cudaSuccess) return cuda_status(e);
        const int64_t rows = cu_seqlens ? T : (int64_t)B * T;
        if (rows > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;  // TMA row coordinate is int32
        const int64_t per_seq = cu_seqlens ? (T + nseq - 1) / nseq : T;
        const int nseg = segments_for(nseq, per_seq, H, current_sms());
        void* ws = nullptr;
        if (nseg > 1) {
            // stream-ordered workspace for the segment maps, start states and map rows,
            // from this library's pool; if it cannot be had, the unsplit kernel computes
            // the same result
            const size_t bytes = kda::chunk_tc_segmented_workspace_bytes(nseq, rows, H, nseg);
            cudaMemPool_t pool = nullptr;
            if (workspace_pool(&pool) != cudaSuccess ||
                cudaMallocFromPoolAsync(&ws, bytes, pool, s) != cudaSuccess) {
                cudaGetLastError();
                ws = nullptr;
            }
        }
        if (ws) {
            g_launches.fetch_add(2, std::memory_order_relaxed);   // three kernels in all
            e = kda::launch_chunk_tc_segmented(q, k, v, alpha, beta, S0, cu_seqlens, (int)nseq,
                                               out, S_final, rows, T, H, nseg, ws, status, s,
                                               fused);
            const cudaError_t ef = cudaFreeAsync(ws, s);
            if (e == cudaSuccess) e = ef;
        } else {
            e = kda::launch_chunk_tc(q, k, v, alpha, beta, S0, cu_seqlens, (int)nseq, out, S_final,
                                     rows, T, H, status, s, nullptr, 0, fused);
        }
        if (e != cudaSuccess) return cuda_status(e);
        return debug_sync() ? kda_device_status(stream) : KDA_OK;
    }
    return cuda_status(kda::launch_chunk_simt(in_bf16, out_bf16, chunk, q, k, v, alpha, beta, S0,
                                              cu_seqlens, (int)nseq, out, S_final, T, H, d_k, d_v,
                                              s));
}

}  // namespace

extern "C" {

kda_status_t kda_forward(const void* q, const void* k, const void* v, const void* alpha,
                         const void* beta, const float* S0, const int32_t* cu_seqlens,
                         int32_t num_seqs, void* out, float* S_final, int32_t B, int64_t T,
                         int32_t H, int32_t d_k, int32_t d_v, int32_t chunk,
                         kda_dtype_t in_dtype, kda_dtype_t out_dtype, kda_stream_t stream) {
    return forward_impl(q, k, v, alpha, beta, S0, cu_seqlens, num_seqs, out, S_final, B, T, H, d_k,
                        d_v, chunk, in_dtype, out_dtype, stream, 0);
}

kda_status_t kda_forward_fused(const void* q, const void* k, const void* v,
                               const void* alpha_logits, const void* beta_logits, const float* S0,
                               const int32_t* cu_seqlens, int32_t num_seqs, void* out,
                               float* S_final, int32_t B, int64_t T, int32_t H, int32_t d_k,
                               int32_t d_v, int32_t chunk, kda_dtype_t in_dtype,
                               kda_dtype_t out_dtype, kda_stream_t stream) {
    return forward_impl(q, k, v, alpha_logits, beta_logits, S0, cu_seqlens, num_seqs, out, S_final,
                        B, T, H, d_k, d_v, chunk, in_dtype, out_dtype, stream, 1);
}

kda_status_t kda_forward_indexed(const void* q, const void* k, const void* v, const void* alpha,
                                 const void* beta, float* S_pool, int32_t num_slots,
                                 const int32_t* slots, const int32_t* cu_seqlens, int32_t num_seqs,
                                 void* out, int32_t B, int64_t T, int32_t H, int32_t d_k,
                                 int32_t d_v, int32_t chunk, kda_dtype_t in_dtype,
                                 kda_dtype_t out_dtype, kda_stream_t stream) {
    if (B < 0 || T < 0 || H <= 0 || num_slots < 0 || !is_dtype(in_dtype) || !is_dtype(out_dtype))
        return KDA_ERR_INVALID_ARG;
    if (cu_seqlens != nullptr && (B != 1 || num_seqs < 0)) return KDA_ERR_INVALID_ARG;
    const int64_t nseq = cu_seqlens ? (int64_t)num_seqs : (int64_t)B;
    if (nseq > 0 && (!S_pool || !slots)) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * T > 0 && (!q || !k || !v || !alpha || !beta || !out)) return KDA_ERR_INVALID_ARG;
    const void* p16[] = {q, k, v, alpha, S_pool, out};
    for (const void* p : p16)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(beta, in_dtype == KDA_BF16 ? 2 : 4) || !aligned_to(cu_seqlens, 4) ||
        !aligned_to(slots, 4))
        return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v)) return KDA_ERR_UNSUPPORTED;
    if (chunk != 16 && chunk != 32 && chunk != 64) return KDA_ERR_UNSUPPORTED;
    if (nseq > 65535 || H > 65535) return KDA_ERR_UNSUPPORTED;
    if (nseq == 0) return KDA_OK;
    g_last_error[0] = '\0';
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (cu_seqlens == nullptr && T <= kMaxStepTokens) {
        // a short multi-token step: the state stays in registers across the T tokens
        if (T == 0) return KDA_OK;   // nothing advances; every state unchanged
        if ((int64_t)B * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
        return cuda_status(kda::launch_decode(in_dtype == KDA_BF16, out_dtype == KDA_BF16, q, k, v,
                                              alpha, beta, S_pool, out, (int64_t)B * H, d_k, d_v,
                                              s, slots, num_slots, H, (int)T));
    }
    if (use_tc(d_k, d_v, chunk, in_dtype, out_dtype)) {
        int* status = nullptr;
        cudaError_t e = device_status_word(&status);
        if (e != cudaSuccess) return cuda_status(e);
        const int64_t rows = cu_seqlens ? T : (int64_t)B * T;
        if (rows > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
        e = kda::launch_chunk_tc(q, k, v, alpha, beta, S_pool, cu_seqlens, (int)nseq, out, S_pool,
                                 rows, T, H, status, s, slots, num_slots);
        if (e != cudaSuccess) return cuda_status(e);
        return debug_sync() ? kda_device_status(stream) : KDA_OK;
    }
    return cuda_status(kda::launch_chunk_simt(in_dtype == KDA_BF16, out_dtype == KDA_BF16, chunk, q,
                                              k, v, alpha, beta, S_pool, cu_seqlens, (int)nseq, out,
                                              S_pool, T, H, d_k, d_v, s, slots, num_slots));
}

kda_status_t kda_decode_step_indexed(const void* q, const void* k, const void* v,
                                     const void* alpha, const void* beta, float* S_pool,
                                     int32_t num_slots, const int32_t* slots, void* out, int32_t N,
                                     int32_t H, int32_t d_k, int32_t d_v, kda_dtype_t in_dtype,
                                     kda_dtype_t out_dtype, kda_stream_t stream) {
    if (N < 0 || H <= 0 || num_slots < 0 || !is_dtype(in_dtype) || !is_dtype(out_dtype))
        return KDA_ERR_INVALID_ARG;
    if (N > 0 && (!q || !k || !v || !alpha || !beta || !S_pool || !slots || !out))
        return KDA_ERR_INVALID_ARG;
    const int es = in_dtype == KDA_BF16 ? 2 : 4;
    if (S_pool && !aligned16(S_pool)) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(q, es) || !aligned_to(k, es) || !aligned_to(v, es) || !aligned_to(alpha, es) ||
        !aligned_to(beta, es) || !aligned_to(out, out_dtype == KDA_BF16 ? 2 : 4) ||
        !aligned_to(slots, 4))
        return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v)) return KDA_ERR_UNSUPPORTED;
    const int64_t NH = (int64_t)N * H;
    if (NH > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (NH == 0) return KDA_OK;
    g_last_error[0] = '\0';
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_status(kda::launch_decode(in_dtype == KDA_BF16, out_dtype == KDA_BF16, q, k, v,
                                          alpha, beta, S_pool, out, NH, d_k, d_v,
                                          reinterpret_cast<cudaStream_t>(stream), slots, num_slots,
                                          H));
}

kda_status_t kda_segment_maps(const void* k, const void* v, const void* alpha, const void* beta,
                              const int32_t* cu_seqlens, int32_t num_seqs, float* maps, int32_t B,
                              int64_t T, int32_t H, int32_t d_k, int32_t d_v, int32_t chunk,
                              kda_dtype_t in_dtype, kda_stream_t stream) {
    if (B < 0 || T < 0 || H <= 0 || !is_dtype(in_dtype)) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens != nullptr && (B != 1 || num_seqs < 0)) return KDA_ERR_INVALID_ARG;
    const int64_t nseq = cu_seqlens ? (int64_t)num_seqs : (int64_t)B;
    if (nseq > 0 && !maps) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * T > 0 && (!k || !v || !alpha || !beta)) return KDA_ERR_INVALID_ARG;
    const void* p16[] = {k, v, alpha, maps};
    for (const void* p : p16)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(beta, 2) || !aligned_to(cu_seqlens, 4)) return KDA_ERR_INVALID_ARG;
    if (!use_tc(d_k, d_v, chunk, in_dtype, KDA_BF16)) {
        std::snprintf(g_last_error, sizeof(g_last_error),
                      "kda_segment_maps: only bf16 inputs, d_k = d_v = 128, chunk 64");
        return KDA_ERR_UNSUPPORTED;
    }
    if (nseq > 65535 || H > 65535) return KDA_ERR_UNSUPPORTED;
    const int64_t rows = cu_seqlens ? T : (int64_t)B * T;
    if (rows > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (nseq == 0) return KDA_OK;
    g_last_error[0] = '\0';
    int* status = nullptr;
    cudaError_t e = device_status_word(&status);
    if (e != cudaSuccess) return cuda_status(e);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    e = kda::launch_segment_maps(k, v, alpha, beta, cu_seqlens, (int)nseq, maps, rows, T, H, status,
                                 reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e);
    return debug_sync() ? kda_device_status(stream) : KDA_OK;
}

kda_status_t kda_segment_scan(const float* S0, const float* maps, int32_t num_maps, float* out,
                              int32_t num_seqs, int32_t H, int32_t d_k, int32_t d_v,
                              kda_stream_t stream) {
    if (num_maps < 0 || num_seqs < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if (d_k != 128 || d_v != 128) return KDA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return KDA_OK;
    if (!out || (num_maps > 0 && !maps)) return KDA_ERR_INVALID_ARG;
    if (!aligned16(out) || (S0 && !aligned16(S0)) || (maps && !aligned16(maps))) return KDA_ERR_INVALID_ARG;
    if (num_seqs > 65535 || H > 65535) return KDA_ERR_UNSUPPORTED;
    g_last_error[0] = '\0';
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_status(kda::launch_apply_maps(S0, maps, num_maps, num_seqs, H, out,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

static kda_status_t decode_impl(const void* q, const void* k, const void* v, const void* alpha,
                             const void* beta, float* S, void* out, int32_t N, int32_t H,
                             int32_t d_k, int32_t d_v, kda_dtype_t in_dtype,
                             kda_dtype_t out_dtype, kda_stream_t stream, int fused) {
    if (N < 0 || H <= 0 || !is_dtype(in_dtype) || !is_dtype(out_dtype))
        return KDA_ERR_INVALID_ARG;
    if (N > 0 && (!q || !k || !v || !alpha || !beta || !S || !out)) return KDA_ERR_INVALID_ARG;
    // S is streamed with 16-byte accesses; the per-token vectors are read element-wise
    const int es = in_dtype == KDA_BF16 ? 2 : 4;
    if (S && !aligned16(S)) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(q, es) || !aligned_to(k, es) || !aligned_to(v, es) || !aligned_to(alpha, es) ||
        !aligned_to(beta, es) || !aligned_to(out, out_dtype == KDA_BF16 ? 2 : 4))
        return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v)) return KDA_ERR_UNSUPPORTED;
    const int64_t NH = (int64_t)N * H;
    if (NH > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (NH == 0) return KDA_OK;
    g_last_error[0] = '\0';
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_status(kda::launch_decode(in_dtype == KDA_BF16, out_dtype == KDA_BF16, q, k, v,
                                          alpha, beta, S, out, NH, d_k, d_v, s, nullptr, 0, H, 1,
                                          fused));
}

kda_status_t kda_decode_step(const void* q, const void* k, const void* v, const void* alpha,
                             const void* beta, float* S, void* out, int32_t N, int32_t H,
                             int32_t d_k, int32_t d_v, kda_dtype_t in_dtype,
                             kda_dtype_t out_dtype, kda_stream_t stream) {
    return decode_impl(q, k, v, alpha, beta, S, out, N, H, d_k, d_v, in_dtype, out_dtype, stream, 0);
}

kda_status_t kda_decode_step_fused(const void* q, const void* k, const void* v,
                                   const void* alpha_logits, const void* beta_logits, float* S,
                                   void* out, int32_t N, int32_t H, int32_t d_k, int32_t d_v,
                                   kda_dtype_t in_dtype, kda_dtype_t out_dtype,
                                   kda_stream_t stream) {
    return decode_impl(q, k, v, alpha_logits, beta_logits, S, out, N, H, d_k, d_v, in_dtype,
                       out_dtype, stream, 1);
}

size_t kda_backward_workspace_bytes(int32_t B, int64_t T, int32_t H, int32_t d_k, int32_t d_v,
                                    int32_t packed, int32_t num_seqs) {
    if (B < 0 || T < 0 || H <= 0 || num_seqs < 0) return 0;
    const int64_t nseq = packed ? (int64_t)num_seqs : (int64_t)B;
    const size_t seq = sizeof(float) * kda::backward_workspace_floats(packed != 0, nseq, T, H, d_k, d_v);
    // enough for either kernel: the dtype is not an argument here
    const size_t tc = d_k == 128 && d_v == 128 ? kda::backward_tc_workspace_bytes(packed != 0, nseq, T, H) : 0;
    return seq > tc ? seq : tc;
}

kda_status_t kda_backward(const void* q, const void* k, const void* v, const void* alpha,
                          const void* beta, const float* S0, const void* dout,
                          const float* dS_final, const int32_t* cu_seqlens, int32_t num_seqs,
                          float* dq, float* dk, float* dv, float* dalpha, float* dbeta,
                          float* dS0, int32_t B, int64_t T, int32_t H, int32_t d_k, int32_t d_v,
                          kda_dtype_t in_dtype, void* workspace, size_t workspace_bytes,
                          kda_stream_t stream) {
    if (B < 0 || T < 0 || H <= 0 || !is_dtype(in_dtype)) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens != nullptr && (B != 1 || num_seqs < 0)) return KDA_ERR_INVALID_ARG;
    const int64_t nseq = cu_seqlens ? (int64_t)num_seqs : (int64_t)B;
    const bool has_tokens = (int64_t)B * T > 0;
    if (has_tokens && (!q || !k || !v || !alpha || !beta || !dout || !dq || !dk || !dv ||
                       !dalpha || !dbeta))
        return KDA_ERR_INVALID_ARG;
    const int es = in_dtype == KDA_BF16 ? 2 : 4;
    const void* elem[] = {q, k, v, alpha, beta, dout};
    for (const void* p : elem)
        if (!aligned_to(p, es)) return KDA_ERR_INVALID_ARG;
    const void* f32[] = {dq, dk, dv, dalpha, dbeta};
    for (const void* p : f32)
        if (!aligned_to(p, 4)) return KDA_ERR_INVALID_ARG;
    const void* vec[] = {S0, dS_final, dS0, workspace};
    for (const void* p : vec)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(cu_seqlens, 4)) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v)) return KDA_ERR_UNSUPPORTED;
    if (nseq * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (nseq == 0) return KDA_OK;
    const bool tc = kda::backward_tc_supported(in_dtype == KDA_BF16, nseq, T, H, d_k, d_v,
                                               cu_seqlens != nullptr);
    const size_t need =
        tc ? kda::backward_tc_workspace_bytes(cu_seqlens != nullptr, nseq, T, H)
           : sizeof(float) * kda::backward_workspace_floats(cu_seqlens != nullptr, nseq, T, H, d_k, d_v);
    // a caller's workspace is held to the documented query (which covers either kernel)
    if (workspace && workspace_bytes < kda_backward_workspace_bytes(
                                           B, T, H, d_k, d_v, cu_seqlens != nullptr, num_seqs))
        return KDA_ERR_INVALID_ARG;
    g_last_error[0] = '\0';
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int* status = nullptr;
    if (tc) {
        cudaError_t e = device_status_word(&status);
        if (e != cudaSuccess) return cuda_status(e);
    }
    float* ws = static_cast<float*>(workspace);
    if (!ws) {
        cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&ws), need, s);
        if (e != cudaSuccess) return cuda_status(e);
    }
    g_launches.fetch_add(tc ? 3 : 1, std::memory_order_relaxed);   // tensor cores: three kernels
    cudaError_t e =
        tc ? kda::launch_backward_tc(q, k, v, alpha, beta, S0, dout, dS_final, cu_seqlens, nseq, T, H,
                                     dq, dk, dv, dalpha, dbeta, dS0, ws, status, s)
           : kda::launch_backward(in_dtype == KDA_BF16, q, k, v, alpha, beta, S0, dout, dS_final,
                                  cu_seqlens, nseq, T, H, d_k, d_v, dq, dk, dv, dalpha, dbeta, dS0,
                                  ws, s);
    if (!workspace) {
        const cudaError_t ef = cudaFreeAsync(ws, s);
        if (e == cudaSuccess) e = ef;
    }
    return cuda_status(e);
}

}  // extern "C"
