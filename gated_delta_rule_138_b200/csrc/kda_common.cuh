// Device helpers shared by the KDA kernels in this directory.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Lower bound of the forget gate: e^-5 rounded to the nearest fp32.  The
// worldcybernews article "Kimi K3 Open Model Surpasses Closed GPT and Anthropic
// Systems on Independent Benchmarks", paragraph 2, holds alpha between e^-5
// and 1 so that BF16 arithmetic neither underflows nor overflows.
constexpr float kAlphaMin = 0x1.b993fep-8f;

// clamp(alpha, e^-5, 1), taken on the fp32 value of the input
__device__ __forceinline__ float clamp_gate(float a) {
    a = a < kAlphaMin ? kAlphaMin : a;
    return a > 1.0f ? 1.0f : a;
}

// Input-side transforms of the fused entry points (plain definitions):
//   alpha = exp(-softplus(x)) = 1 / (1 + e^x),   beta = sigmoid(x) = 1 / (1 + e^-x).
// exp overflows to +inf for large x and the (fast, approximate) reciprocal then gives 0,
// the limit.
__device__ __forceinline__ float gate_from_logit(float x) { return __fdividef(1.0f, 1.0f + __expf(x)); }
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);  // round to nearest even
}

// Sequence n's token range [bos, bos + len) in the flattened [B*T] token axis.
// A packed table is clamped into [0, T] so a malformed one cannot send a
// kernel out of bounds.
__device__ __forceinline__ void seq_range(const int32_t* __restrict__ cu_seqlens, int n, int64_t T,
                                          int64_t& bos, int64_t& len) {
    if (cu_seqlens == nullptr) {
        bos = (int64_t)n * T;
        len = T;
        return;
    }
    int64_t a = cu_seqlens[n], b = cu_seqlens[n + 1];
    a = a < 0 ? 0 : (a > T ? T : a);
    b = b < a ? a : (b > T ? T : b);
    bos = a;
    len = b - a;
}

// Chunks of C tokens before sequence n (the sum of ceil(len_m / C) over m < n),
// computed by one whole warp; every lane returns the total.
__device__ __forceinline__ int64_t chunks_before(const int32_t* __restrict__ cu, int n, int64_t T,
                                                 int C) {
    if (cu == nullptr) return (int64_t)n * ((T + C - 1) / C);
    int64_t acc = 0;
    for (int m = (int)(threadIdx.x & 31); m < n; m += 32) {
        int64_t b, l;
        seq_range(cu, m, T, b, l);
        acc += (l + C - 1) / C;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
}

// Longest-first schedule for packed batches: CTAs are launched in blockIdx.z
// order, so z-th CTA column takes the sequence of rank z in decreasing length
// (ties by index).  Each CTA ranks the lengths itself from cu_seqlens: no
// workspace, O(num_seqs^2) work, used only up to kMaxRankedSeqs sequences.
constexpr int kMaxRankedSeqs = 1024;
__device__ __forceinline__ int64_t seq_len_at(const int32_t* __restrict__ cu, int i, int64_t T) {
    int64_t a = cu[i], b = cu[i + 1];
    a = a < 0 ? 0 : (a > T ? T : a);
    b = b < a ? a : (b > T ? T : b);
    return b - a;
}
// Warp-collective (call from one full warp): the sequence of rank z.
__device__ __forceinline__ int longest_first_seq(const int32_t* __restrict__ cu, int nseq, int z,
                                                 int64_t T) {
    if (cu == nullptr || nseq > kMaxRankedSeqs) return z;
    const int lane = threadIdx.x & 31;
    int found = -1;
    for (int i = lane; i < nseq; i += 32) {
        const int64_t li = seq_len_at(cu, i, T);
        int rank = 0;
        for (int j = 0; j < nseq; ++j) {
            const int64_t lj = seq_len_at(cu, j, T);
            rank += (lj > li) || (lj == li && j < i);
        }
        if (rank == z) found = i;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) found = max(found, __shfl_xor_sync(0xffffffffu, found, o));
    return found < 0 ? z : found;
}

}  // namespace kda
