// KDA backward pass on the sm_100a tensor cores (bf16 inputs, d_k = d_v = 128, C = 64),
// chunk-parallel: the reverse mode of the chunk form of the forward.
//
// The worldcybernews article "Kimi K3 Open Model Surpasses Closed GPT and Anthropic
// Systems on Independent Benchmarks", paragraph 2, gives the recurrence
// S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t;
// paragraph 3 processes a chunk's tokens in parallel and carries the state across
// chunks.  The pages print no backward; this is the reverse mode of that forward.
// Per chunk, with start state S0 and the forward's tiles (kda_bwd_record.cuh):
//
//   R = V - (k*gamma) S0,  U = T diag(beta) R,  O = (q*gamma) S0 + P U,
//   S_end = Diag(gamma_C) S0 + (k*eta)^T U,
//   [A/beta ; P] = [k*lam ; q*lam] [k*rho^0 ; k*rho^1]^T   (A strictly, P weakly lower)
//
// and, for a loss with dO = dL/dO and dS = dL/dS_end:
//
//   dU = P^T dO + (k*eta) dS,   dY = T^T dU,   dR = beta dY (= dV)
//   dS0 = Diag(gamma_C) dS + (q*gamma)^T dO - (k*gamma)^T dR          (the only chain)
//   dA = -strict(dY U^T),  dP = lower(dO U^T)
//   G = [beta dA ; dP] laid out like [A/beta ; P] (sub-chunk I's rows in I's columns)
//   [d(k*lam) ; d(q*lam)] = G [k*rho^0 ; k*rho^1],   [d(k*rho^0) ; d(k*rho^1)] = G^T [k*lam ; q*lam]
//   d(k*gamma) = -dR S0^T,  d(q*gamma) = dO S0^T,  d(k*eta) = U dS^T
//   dbeta = rowsum(R * dY) + rowsum(dA * A/beta)
//
// dk, dq are those operand gradients times their decay factors, and the gradient of
// the log-gates sums each operand times its gradient: for token s and key channel c,
//   dlog a_s = sum_{r >= s} (Kt dKt + Qt dQt + L dL + Lq dLq - R0 dR0 - R1 dR1)_r
//            + sum_{j < s} (Kh dKh)_j + gamma_C sum_n S0 dS
// (the sub-chunk reference terms cancel between the left and right factors), and
// dalpha = dlog a / a where e^-5 <= alpha <= 1, else 0.  The left/right pair terms
// (L dL, Lq dLq, R dR) are taken against the same bf16 tile values that the MMAs
// read: the two ends of a pair then cancel exactly, and the products stay bf16.
//
// Three passes: the forward kernel in record mode writes the records; the state
// gradient kernel below walks each (sequence, head) backwards, carrying dS in TMEM,
// and writes dv, the first part of dbeta, dS0 and the records' dS and dY; the chunk
// kernel then takes every (chunk, head) in parallel.
#include <cuda.h>

#include "kda_bwd_record.cuh"
#include "kda_common.cuh"
#include "kda_sm100.cuh"
#include "kda_tc_maps.cuh"

// Optional phase-boundary hook of the chunk kernel for profiling builds (no-op in the library).
#ifndef KDA_BWD_PHASE
#define KDA_BWD_PHASE(i)
#endif

namespace kda {
using namespace sm100;

namespace bwdtc {

constexpr int C = 64, DK = 128, DV = 128;
constexpr int NT = 256;                 // eight compute warps
constexpr uint64_t kWaitNs = 2000000000ull;

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
    return row * 128u + (((chunk ^ row) & 7u) << 4);
}
__device__ __forceinline__ uint4 pack8(const float* v) {
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
}
__device__ __forceinline__ void unpack8(uint4 raw, float* v) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
// bf16 element (row, col) of a tile of 64-column swizzled atoms of `atom` bytes
__device__ __forceinline__ float tile_at(const uint8_t* t, uint32_t atom, int row, int col) {
    const uint8_t* p = t + (uint32_t)(col >> 6) * atom + swz((uint32_t)row, (uint32_t)((col & 63) >> 3)) +
                       (uint32_t)(col & 7) * 2u;
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
    tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(&v[0]));
    tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
    tmem_ld16(taddr + 32, *reinterpret_cast<float(*)[16]>(&v[32]));
    tmem_ld16(taddr + 48, *reinterpret_cast<float(*)[16]>(&v[48]));
    tmem_wait_ld();
}
__device__ __forceinline__ void sync_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// K-major operand, 64-column atoms of `atom` bytes: the descriptor of K step ks (16 elements)
__device__ __forceinline__ uint64_t kmaj(uint32_t base, uint32_t atom, int ks) {
    return sdesc_sw128(base + (uint32_t)(ks >> 2) * atom + (uint32_t)(ks & 3) * 32u);
}
// MN-major operand (rows = K), 64-wide MN atoms of `atom` bytes: K step ks (16 rows)
__device__ __forceinline__ uint64_t mnmaj(uint32_t base, uint32_t atom, int ks) {
    return sdesc_sw128(base + (uint32_t)ks * 2048u, 1024, atom);
}

// ================================================================ state gradient pass
//
// One CTA per (sequence, head), chunks from the last: eight compute warps and one
// control warp whose lane 0 issues every copy and MMA.  TMEM: dS fp32 [0, 128),
// dU (M = 64) [128, 256), dY (M = 64) [256, 384).
namespace ds {
constexpr uint32_t OFF_DS = 0;          // dS bf16 [128 c][128 n], MN-major B (two [128][64] atoms)
constexpr uint32_t OFF_P = 32768;       // P [64 r][64 j]
constexpr uint32_t OFF_KH = 40960;      // k*eta [64 j][128 c]
constexpr uint32_t OFF_T = 57344;       // T [64 j][64 m]
constexpr uint32_t OFF_QT = 65536;      // q*gamma [64 r][128 c]
constexpr uint32_t OFF_KT = 81920;      // k*gamma [64 r][128 c]
constexpr uint32_t OFF_DO = 98304;      // dO [64 r][128 n] (TMA), chunk parity 0; parity 1 at OFF_DO1
constexpr uint32_t OFF_RV = 114688;     // R = V - (k*gamma) S0 [64 j][128 n], chunk parity 0; 1 at OFF_RV1
constexpr uint32_t OFF_DU = 131072;     // dU bf16 [64 j][128 n], MN-major B
constexpr uint32_t OFF_MDR = 147456;    // -dR bf16 [64 r][128 n], MN-major B
constexpr uint32_t OFF_DY = 163840;     // dY bf16 [64 m][128 n] (to the record)
constexpr uint32_t OFF_DO1 = 180224;
constexpr uint32_t OFF_RV1 = 196608;
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t M_GC = 0;            // float [2 parities][128]
constexpr uint32_t M_BETA = 1024;       // float [64]
constexpr uint32_t M_DB = 1280;         // float [64][2]
constexpr uint32_t M_BAR = 1792;        // uint64 x4: loads A (P, k*eta, dO, gamma_C, R), B (T), C (q*gamma, k*gamma), MMA
constexpr uint32_t M_TMEM = 1824;
constexpr uint32_t M_FLAG = 1828;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 1856 + 1024;
constexpr uint32_t TM_DS = 0, TM_DU = 128, TM_DY = 256;
}  // namespace ds

// 32 consecutive fp32 TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(&v[0]));
    tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
    tmem_wait_ld();
}

__global__ void __launch_bounds__(NT + 32, 1)
kda_bwd_dstate_kernel(const __grid_constant__ CUtensorMap tmDO, const __nv_bfloat16* __restrict__ beta,
                      const float* __restrict__ dS_final, const int32_t* __restrict__ cu_seqlens,
                      int64_t T, int H, uint8_t* __restrict__ rec, int64_t rec_chunks,
                      float* __restrict__ dv, float* __restrict__ dbeta, float* __restrict__ dS0,
                      int* status) {
    using namespace ds;
    extern __shared__ uint8_t smem_raw[];
    // the 1024-aligned base as an offset into the shared array (the compiler keeps
    // every access below a shared-memory one)
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* sGC = reinterpret_cast<float*>(sm + OFF_MISC + M_GC);
    float* sBeta = reinterpret_cast<float*>(sm + OFF_MISC + M_BETA);
    float* sDB = reinterpret_cast<float*>(sm + OFF_MISC + M_DB);
    uint64_t* barA = reinterpret_cast<uint64_t*>(sm + OFF_MISC + M_BAR);
    uint64_t* barB = barA + 1;
    uint64_t* barC = barA + 2;
    uint64_t* barM = barA + 3;
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC + M_TMEM);
    int* sFlag = reinterpret_cast<int*>(sm + OFF_MISC + M_FLAG);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool compute = warp < NT / 32;
    const bool ctl = warp == NT / 32 && lane == 0;
    const int q4 = warp & 3, hf = (warp >> 2) & 1;
    const int h = blockIdx.y;
    __shared__ int s_seq;
    __shared__ int64_t s_cbase;
    if (threadIdx.x < 32) {
        const int sq = longest_first_seq(cu_seqlens, (int)gridDim.z, (int)blockIdx.z, T);
        const int64_t cb = chunks_before(cu_seqlens, sq, T, C);
        if (threadIdx.x == 0) { s_seq = sq; s_cbase = cb; }
    }
    __syncthreads();
    const int n = s_seq;
    int64_t bos, len;
    seq_range(cu_seqlens, n, T, bos, len);
    int nchunks = (int)((len + C - 1) / C);
    if (s_cbase + nchunks > rec_chunks)   // a malformed packed table: cut at the records' end
        nchunks = (int)max((int64_t)0, rec_chunks - s_cbase);
    auto rec_of = [&](int i) { return rec + ((size_t)(s_cbase + i) * H + h) * bwdrec::BYTES; };
    auto dO_of = [&](int i) { return sm + ((i & 1) ? OFF_DO1 : OFF_DO); };
    auto rv_of = [&](int i) { return sm + ((i & 1) ? OFF_RV1 : OFF_RV); };

    if (tid == 0) {
        mbar_init(barA, 1);
        mbar_init(barB, 1);
        mbar_init(barC, 1);
        mbar_init(barM, 1);
        mbar_fence_init();
        *sFlag = 0;
    }
    if (warp == 0) tmem_alloc(sTmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t tlane = (uint32_t)(32 * q4) << 16;

    // dS = dL/dS_final (or 0): TMEM fp32 and its bf16 copy
    if (compute) {
        const int c = 32 * q4 + lane;
        const float* src = dS_final ? dS_final + (((size_t)n * H + h) * DK + c) * DV + 64 * hf : nullptr;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
                const float4 f = src ? *reinterpret_cast<const float4*>(src + 16 * blk + i)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                v[i] = f.x; v[i + 1] = f.y; v[i + 2] = f.z; v[i + 3] = f.w;
            }
            tmem_st16(tmem + tlane + TM_DS + 64 * hf + 16 * blk, v);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
                *reinterpret_cast<uint4*>(sm + OFF_DS + hf * 16384 + swz(c, 2 * blk + ch)) =
                    pack8(&v[8 * ch]);
        }
        tmem_wait_st();
    }

    uint32_t phA = 0, phB = 0, phC = 0, phM = 0;
    uint32_t nA = 0, nB = 0, nC = 0;   // (control thread) copies issued per stream
    bool mma_out = false;
    uint32_t mma_out_ph = 0;
    bool ok = true;
    auto wait_bar = [&](uint64_t* bar, uint32_t& ph) {
        if (ok && !mbar_wait_ns(bar, ph, kWaitNs)) ok = false;
        ph ^= 1u;
    };
    auto commit = [&]() {
        mma_commit(barM);
        mma_out = true;
        mma_out_ph = phM;
    };
    auto wait_mma = [&]() {
        if (ok) {
            if (mbar_wait_ns(barM, phM, kWaitNs)) mma_out = false;
            else ok = false;
        }
        phM ^= 1u;
        tc_fence_after();
    };
    // loads a chunk ahead where the buffers allow: A (needed first) lands while the
    // previous chunk's dY and dS steps run
    auto issue_a = [&](int i) {
        uint8_t* rp = rec_of(i);
        const int64_t row0 = bos + (int64_t)i * C;
        mbar_arrive_expect_tx(barA, 8192 + 16384 + 16384 + 16384 + 512);
        bulk_load(sm + OFF_P, rp + bwdrec::P, 8192, barA);
        bulk_load(sm + OFF_KH, rp + bwdrec::KH, 16384, barA);
        bulk_load(rv_of(i), rp + bwdrec::RV, 16384, barA);
        bulk_load(sGC + 128 * (i & 1), rp + bwdrec::GC, 512, barA);
#pragma unroll
        for (int a = 0; a < 2; ++a)
            tma_load_2d(dO_of(i) + a * 8192, &tmDO, barA, h * DV + 64 * a, (int)row0);
        ++nA;
    };
    auto issue_b = [&](int i) {
        mbar_arrive_expect_tx(barB, 8192);
        bulk_load(sm + OFF_T, rec_of(i) + bwdrec::T, 8192, barB);
        ++nB;
    };
    auto issue_c = [&](int i) {
        uint8_t* rp = rec_of(i);
        mbar_arrive_expect_tx(barC, 2 * 16384);
        bulk_load(sm + OFF_QT, rp + bwdrec::QT, 16384, barC);
        bulk_load(sm + OFF_KT, rp + bwdrec::KT, 16384, barC);
        ++nC;
    };
    if (ctl && nchunks > 0) {
        issue_a(nchunks - 1);
        issue_b(nchunks - 1);
        issue_c(nchunks - 1);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    bool broke = false;
    for (int i = nchunks - 1; i >= 0; --i) {
        const int64_t row0 = bos + (int64_t)i * C;
        const int Lc = (int)((len - (int64_t)i * C) < C ? (len - (int64_t)i * C) : C);
        float bval = 0.0f;
        if (compute && tid < C && tid < Lc) bval = __bfloat162float(beta[(size_t)(row0 + tid) * H + h]);

        // ---- dU = P^T dO + (k*eta) dS (the dS copy is in place)
        if (ctl) {
            wait_bar(barA, phA);
            if (ok) {
                bulk_store(rec_of(i) + bwdrec::DS, sm + OFF_DS, 32768);
                bulk_commit_group();
                constexpr uint32_t id64 = idesc_bf16(64, 128, true, true);
                constexpr uint32_t id64k = idesc_bf16(64, 128, false, true);
                const uint32_t p0 = smem_u32(sm + OFF_P), d0 = smem_u32(dO_of(i));
                const uint32_t kh = smem_u32(sm + OFF_KH), s0 = smem_u32(sm + OFF_DS);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_DU, mnmaj(p0, 8192, ks), mnmaj(d0, 8192, ks), id64, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tmem + TM_DU, kmaj(kh, 8192, ks), mnmaj(s0, 16384, ks), id64k, 1);
                bulk_wait_read_all();   // the dS copy is rewritten at the end of this chunk
                commit();
            }
            wait_mma();
        }
        if (compute) {
            wait_bar(barA, phA);   // gamma_C
            wait_mma();
            const int c = 32 * q4 + lane;
            // dS <- Diag(gamma_C) dS in TMEM (the MMAs read the bf16 copy)
            const float g = sGC[128 * (i & 1) + c];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const uint32_t ta = tmem + tlane + TM_DS + 64 * hf + 32 * p;
                float v[32];
                tmem_ld32(ta, v);
#pragma unroll
                for (int k2 = 0; k2 < 32; ++k2) v[k2] *= g;
                tmem_st16(ta, *reinterpret_cast<float(*)[16]>(&v[0]));
                tmem_st16(ta + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
            }
            tmem_wait_st();
            // dU as the MN-major B operand: M=64 row j = 16 q4 + lane (lane < 16)
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float v[32];
                tmem_ld32(tmem + tlane + TM_DU + 64 * hf + 32 * p, v);
                if (lane < 16) {
                    const int j = 16 * q4 + lane;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch)
                        *reinterpret_cast<uint4*>(sm + OFF_DU + hf * 8192 + swz(j, 4 * p + ch)) =
                            pack8(&v[8 * ch]);
                }
            }
            if (tid < C) sBeta[tid] = bval;
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- dY = T^T dU
        if (ctl) {
            // every thread has passed its wait on this chunk's A loads: P and k*eta are
            // consumed, and the other dO, gamma_C and R buffers are free (the previous
            // chunk's R was last read before its dS step)
            if (i > 0 && ok) issue_a(i - 1);
            wait_bar(barB, phB);
            if (ok) {
                constexpr uint32_t id64 = idesc_bf16(64, 128, true, true);
                const uint32_t t0 = smem_u32(sm + OFF_T), u0 = smem_u32(sm + OFF_DU);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_DY, mnmaj(t0, 8192, ks), mnmaj(u0, 8192, ks), id64, ks > 0);
                commit();
            }
            wait_mma();
            if (i > 0 && ok) issue_b(i - 1);   // T is consumed
        }
        if (compute) {
            wait_mma();
            const int m = 16 * q4 + lane;
            const float b = lane < 16 ? sBeta[m] : 0.0f;
            float part = 0.0f;
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float v[32];
                tmem_ld32(tmem + tlane + TM_DY + 64 * hf + 32 * p, v);
                if (lane < 16) {
                    // dV = dR = beta dY (fp32 out), -dR and dY as bf16 tiles, dbeta's first part
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        float r8[8], w[8];
                        const uint32_t off = hf * 8192 + swz(m, 4 * p + ch);
                        unpack8(*reinterpret_cast<const uint4*>(rv_of(i) + off), r8);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            part = fmaf(r8[e], v[8 * ch + e], part);
                            w[e] = -b * v[8 * ch + e];
                        }
                        *reinterpret_cast<uint4*>(sm + OFF_MDR + off) = pack8(w);
                        *reinterpret_cast<uint4*>(sm + OFF_DY + off) = pack8(&v[8 * ch]);
                    }
                    if (m < Lc) {
                        float* dst = dv + ((size_t)(row0 + m) * H + h) * DV + 64 * hf + 32 * p;
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4*>(dst + e) =
                                make_float4(b * v[e], b * v[e + 1], b * v[e + 2], b * v[e + 3]);
                    }
                }
            }
            if (lane < 16) sDB[2 * m + hf] = part;
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- dS += (q*gamma)^T dO - (k*gamma)^T dR
        if (ctl) {
            wait_bar(barC, phC);
            if (ok) {
                bulk_store(rec_of(i) + bwdrec::DY, sm + OFF_DY, 16384);
                bulk_commit_group();
                constexpr uint32_t id128 = idesc_bf16(128, 128, true, true);
                const uint32_t qt = smem_u32(sm + OFF_QT), kt = smem_u32(sm + OFF_KT);
                const uint32_t d0 = smem_u32(dO_of(i)), r0 = smem_u32(sm + OFF_MDR);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_DS, mnmaj(qt, 8192, ks), mnmaj(d0, 8192, ks), id128, 1);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_DS, mnmaj(kt, 8192, ks), mnmaj(r0, 8192, ks), id128, 1);
                bulk_wait_read_all();   // dY's tile is rewritten next chunk
                commit();
            }
            wait_mma();
            if (i > 0 && ok) issue_c(i - 1);   // q*gamma and k*gamma are consumed
        }
        if (compute) {
            if (tid < C && tid < Lc)
                dbeta[(size_t)(row0 + tid) * H + h] = sDB[2 * tid] + sDB[2 * tid + 1];
            wait_mma();
            // the new dS's bf16 copy for the next chunk's MMAs
            const int c = 32 * q4 + lane;
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float v[32];
                tmem_ld32(tmem + tlane + TM_DS + 64 * hf + 32 * p, v);
#pragma unroll
                for (int ch = 0; ch < 4; ++ch)
                    *reinterpret_cast<uint4*>(sm + OFF_DS + hf * 16384 + swz(c, 4 * p + ch)) =
                        pack8(&v[8 * ch]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        const int any_timeout = __syncthreads_or(!ok);
        tc_fence_after();
        if (any_timeout) {
            broke = true;
            break;
        }
    }

    if (!ok) atomicExch(sFlag, 1);
    __syncthreads();
    if (ctl) {
        bulk_wait_all();
        if (*sFlag) {   // let this CTA's own copies and MMAs in flight finish (bounded)
            if (nA) mbar_wait_ns(barA, (nA - 1) & 1u, kWaitNs);
            if (nB) mbar_wait_ns(barB, (nB - 1) & 1u, kWaitNs);
            if (nC) mbar_wait_ns(barC, (nC - 1) & 1u, kWaitNs);
            if (mma_out) mbar_wait_ns(barM, mma_out_ph, kWaitNs);
        }
    }
    __syncthreads();
    if (*sFlag) {
        if (tid == 0) atomicExch(status, 1);
    } else if (compute && dS0 && !broke) {
        const int c = 32 * q4 + lane;
        float* dst = dS0 + (((size_t)n * H + h) * DK + c) * DV + 64 * hf;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            float v[32];
            tmem_ld32(tmem + tlane + TM_DS + 64 * hf + 32 * p, v);
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(dst + 32 * p + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ================================================================ chunk gradient pass
//
// One CTA per (chunk, head), all in parallel.  Thread 0 issues the copies and MMAs;
// eight warps do the element-wise work.  Products, in three groups:
//   1: [dY ; dO] U^T (dA and dP rows, M=128 N=64), [A/beta ; P] again (M=128 N=96),
//      (k*eta) gradient transposed: dS U^T (M=128 c, N=64 j)
//   2: the state terms transposed, S0 [dR ; dO]^T (M=128 c, N=128: -dKt then dQt),
//      the left-factor gradients transposed, R^T G^T (M=128 c, N=128: dL then dLq),
//      the right-factor gradients transposed, L^T G (M=128 c, N=128: dR0 then dR1)
// so that every gradient of group 2 and the (k*eta) one have key channel c in TMEM
// lane c: one thread per channel then walks the chunk's tokens for dq, dk and dalpha.
namespace ck {
constexpr uint32_t OFF_STK = 0;         // [dY ; dO] then [dR ; dO]: [128][128 n] (two [128][64] atoms)
constexpr uint32_t OFF_S0 = 32768;      // S0 bf16 [128 c][128 n]
constexpr uint32_t OFF_L = 65536;       // [k*lam ; q*lam] [128 r][128 c]
constexpr uint32_t OFF_R = 98304;       // [k*rho^0 ; k*rho^1] [96][128 c] (two [96][64] atoms)
constexpr uint32_t OFF_U = 122880;      // U [64 j][128 n]
constexpr uint32_t OFF_DS = 139264;     // dS bf16 [128 c][128 n]
constexpr uint32_t OFF_G = 122880;      // G [128 r][128 col] (two [128][64] atoms), over U and dS
constexpr uint32_t OFF_AL = 172032;     // alpha [64 r][128 c] (TMA)
constexpr uint32_t OFF_Q = 188416;      // q [64 r][128 c] (TMA)
constexpr uint32_t OFF_K = 204800;      // k [64 r][128 c] (TMA)
constexpr uint32_t OFF_MISC = 221184;
constexpr uint32_t M_GC = 0;            // float [128] gamma_C
constexpr uint32_t M_BETA = 512;        // float [64]
constexpr uint32_t M_DGC = 768;         // float [2][128] gamma_C * sum_n S0 dS, two halves
constexpr uint32_t M_DB = 1792;         // float [64][2] dbeta's second part, two halves
constexpr uint32_t M_TOT = 2304;        // float [2 halves][2 (X, Y)][128]
constexpr uint32_t M_BAR = 4352;        // uint64 x3: loads A (group 1's operands), loads B, MMA
constexpr uint32_t M_TMEM = 4376;
constexpr uint32_t M_FLAG = 4380;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 4384 + 1024;
constexpr uint32_t TM_G1 = 0, TM_AP = 64, TM_KH = 160, TM_ST = 224, TM_LF = 352, TM_RF = 0;
}  // namespace ck

__global__ void __launch_bounds__(NT, 1)
kda_bwd_chunk_kernel(const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __nv_bfloat16* __restrict__ beta, int H, const uint8_t* __restrict__ rec,
                     const bwdrec::Header* __restrict__ hdr, float* __restrict__ dq,
                     float* __restrict__ dk, float* __restrict__ dalpha, float* __restrict__ dbeta,
                     int* status) {
    using namespace ck;
    const int64_t chunk = blockIdx.x;
    const int h = blockIdx.y;
    const bwdrec::Header hd = hdr[chunk];
    if (hd.len <= 0) return;   // uniform: no such chunk
    const int64_t row0 = hd.row0;
    const int Lc = hd.len < C ? hd.len : C;
    const uint8_t* rp = rec + ((size_t)chunk * H + h) * bwdrec::BYTES;

    extern __shared__ uint8_t smem_raw[];
    // the 1024-aligned base as an offset into the shared array (the compiler keeps
    // every access below a shared-memory one)
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* sGC = reinterpret_cast<float*>(sm + OFF_MISC + M_GC);
    float* sBeta = reinterpret_cast<float*>(sm + OFF_MISC + M_BETA);
    float* sDGC = reinterpret_cast<float*>(sm + OFF_MISC + M_DGC);
    float* sDB = reinterpret_cast<float*>(sm + OFF_MISC + M_DB);
    float* sTot = reinterpret_cast<float*>(sm + OFF_MISC + M_TOT);
    uint64_t* barL = reinterpret_cast<uint64_t*>(sm + OFF_MISC + M_BAR);
    uint64_t* barL2 = barL + 1;
    uint64_t* barM = barL + 2;
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC + M_TMEM);
    int* sFlag = reinterpret_cast<int*>(sm + OFF_MISC + M_FLAG);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, hf = warp >> 2;
    const bool issuer = tid == 0;

    if (issuer) {
        mbar_init(barL, 1);
        mbar_init(barL2, 1);
        mbar_init(barM, 1);
        mbar_fence_init();
        *sFlag = 0;
    }
    if (warp == 0) tmem_alloc(sTmem, 512);
    tc_fence_before();
    __syncthreads();
    KDA_BWD_PHASE(0);
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t tlane = (uint32_t)(32 * q4) << 16;

    if (issuer) {
        // A: what group 1's first products read (dY, dO, U, dS); B: the rest
        mbar_arrive_expect_tx(barL, 16384 + 16384 + 16384 + 32768);
        bulk_load(sm + OFF_STK, rp + bwdrec::DY, 8192, barL);   // dY: rows 0..63 of both atoms
        bulk_load(sm + OFF_STK + 16384, rp + bwdrec::DY + 8192, 8192, barL);
#pragma unroll
        for (int a = 0; a < 2; ++a)
            tma_load_2d(sm + OFF_STK + a * 16384 + 8192, &tmDO, barL, h * DV + 64 * a, (int)row0);
        bulk_load(sm + OFF_U, rp + bwdrec::U, 16384, barL);
        bulk_load(sm + OFF_DS, rp + bwdrec::DS, 32768, barL);
        mbar_arrive_expect_tx(barL2, 32768 + 32768 + 24576 + 512 + 3 * 16384);
        bulk_load(sm + OFF_S0, rp + bwdrec::S, 32768, barL2);
        bulk_load(sm + OFF_L, rp + bwdrec::L, 32768, barL2);
        bulk_load(sm + OFF_R, rp + bwdrec::R, 24576, barL2);
        bulk_load(sGC, rp + bwdrec::GC, 512, barL2);
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            tma_load_2d(sm + OFF_AL + a * 8192, &tmA, barL2, h * DK + 64 * a, (int)row0);
            tma_load_2d(sm + OFF_Q + a * 8192, &tmQ, barL2, h * DK + 64 * a, (int)row0);
            tma_load_2d(sm + OFF_K + a * 8192, &tmK, barL2, h * DK + 64 * a, (int)row0);
        }
    }
    float bval = 0.0f;
    if (tid < C && tid < Lc) bval = __bfloat162float(beta[(size_t)(row0 + tid) * H + h]);

    bool ok = true;
    uint32_t phL = 0, phM = 0;
    bool mma_out = false;
    uint32_t mma_out_ph = 0;
    auto wait_mma = [&]() {
        if (ok) {
            if (mbar_wait_ns(barM, phM, kWaitNs)) mma_out = false;
            else ok = false;
        }
        phM ^= 1u;
        tc_fence_after();
    };
    if (!mbar_wait_ns(barL, phL, kWaitNs)) ok = false;
    KDA_BWD_PHASE(1);

    // ---- group 1: [dY ; dO] U^T and dS U^T on loads A, [A/beta ; P] once B has landed
    if (issuer && ok) {
        const uint32_t stk = smem_u32(sm + OFF_STK), u0 = smem_u32(sm + OFF_U);
        const uint32_t ds0 = smem_u32(sm + OFF_DS);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_G1, kmaj(stk, 16384, ks), kmaj(u0, 8192, ks), idesc_bf16(128, 64), ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_KH, kmaj(ds0, 16384, ks), kmaj(u0, 8192, ks), idesc_bf16(128, 64), ks > 0);
    }
    if (ok && !mbar_wait_ns(barL2, phL, kWaitNs)) ok = false;
    phL ^= 1u;
    if (issuer && ok) {
        const uint32_t l0 = smem_u32(sm + OFF_L), r0 = smem_u32(sm + OFF_R);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_AP, kmaj(l0, 16384, ks), kmaj(r0, 12288, ks), idesc_bf16(128, 96), ks > 0);
    }
    if (issuer && ok) {   // one commit covers the group (MMAs of one thread complete in order)
        mma_commit(barM);
        mma_out = true;
        mma_out_ph = phM;
    }
    // meanwhile: gamma_C sum_n S0 dS per key channel (two halves of n), beta
    {
        const int c = tid & 127, half = tid >> 7;
        float acc = 0.0f;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            float a8[8], b8[8];
            unpack8(*reinterpret_cast<const uint4*>(sm + OFF_S0 + half * 16384 + swz(c, ch)), a8);
            unpack8(*reinterpret_cast<const uint4*>(sm + OFF_DS + half * 16384 + swz(c, ch)), b8);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(a8[e], b8[e], acc);
        }
        sDGC[half * 128 + c] = acc * sGC[c];
        if (tid < C) sBeta[tid] = bval;
    }
    __syncthreads();   // dS is no longer read by the CUDA cores (G goes over it)
    wait_mma();
    KDA_BWD_PHASE(2);

    // ---- G = [beta dA ; dP] in the column layout of [A/beta ; P]; dbeta's second part;
    //      [dY ; dO] -> [dR ; dO]
    {
        const int R = 32 * q4 + lane, r = R & 63, j0 = 32 * hf;
        const bool arow = R < 64;
        float v[32];
        tmem_ld16(tmem + tlane + TM_G1 + j0, *reinterpret_cast<float(*)[16]>(&v[0]));
        tmem_ld16(tmem + tlane + TM_G1 + j0 + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
        tmem_wait_ld();
        float w[32];
        const bool live = r < Lc;
        if (arow) {
            // dA[r][j] = -(dY U^T)[r][j] for j < r; A/beta's columns for row r: j (r < 32)
            // or 32 + j (r >= 32)
            // (warp-uniform: rows r < 32 are warp quarter 0, whose j >= 32 half is all zero)
            float m[32];
            const bool wneed = !(q4 == 0 && hf == 1);
            if (wneed) {
                const uint32_t col = (q4 == 0 ? 0u : 32u) + (uint32_t)j0;
                tmem_ld16(tmem + tlane + TM_AP + col, *reinterpret_cast<float(*)[16]>(&m[0]));
                tmem_ld16(tmem + tlane + TM_AP + col + 16, *reinterpret_cast<float(*)[16]>(&m[16]));
                tmem_wait_ld();
            }
            const bool need = live && wneed;
            const float b = sBeta[r];
            float part = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float da = (need && j0 + i < r) ? -v[i] : 0.0f;
                if (need) part = fmaf(da, m[i], part);
                w[i] = b * da;
            }
            sDB[2 * r + hf] = part;
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = (live && j0 + i <= r) ? v[i] : 0.0f;
        }
        // row R of G: columns j (r < 32) or 32 + j (r >= 32); the rest zero
        uint8_t* g = sm + OFF_G;
        const float z8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (hf == 0) {   // columns 0..63 (atom 0)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const bool val = (r < 32) ? (ch < 4) : (ch >= 4);
                const float* src = val ? &w[8 * (ch & 3)] : z8;
                *reinterpret_cast<uint4*>(g + swz(R, ch)) = pack8(src);
            }
        } else {         // columns 64..127 (atom 1): j = 32..63 of rows r >= 32 at 64..95
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const bool val = r >= 32 && ch < 4;
                const float* src = val ? &w[8 * ch] : z8;
                *reinterpret_cast<uint4*>(g + 16384 + swz(R, ch)) = pack8(src);
            }
        }
        // dY rows -> dR = beta dY (rows 0..63 of the stacked tile)
        {
            const int e = tid;                 // 256 threads x 4 pieces of 16 bytes
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const int idx = e + NT * p;    // 0..1023: (row 0..63, atom 0..1, chunk 0..7)
                const int row = idx >> 4, a = (idx >> 3) & 1, ch = idx & 7;
                uint8_t* ptr = sm + OFF_STK + a * 16384 + swz(row, ch);
                float y8[8];
                unpack8(*reinterpret_cast<const uint4*>(ptr), y8);
                const float b = sBeta[row];
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2) y8[k2] *= b;
                *reinterpret_cast<uint4*>(ptr) = pack8(y8);
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    KDA_BWD_PHASE(3);
    tc_fence_after();

    // ---- group 2
    if (issuer && ok) {
        const uint32_t s0 = smem_u32(sm + OFF_S0), stk = smem_u32(sm + OFF_STK);
        const uint32_t l0 = smem_u32(sm + OFF_L), r0 = smem_u32(sm + OFF_R);
        const uint32_t g0 = smem_u32(sm + OFF_G);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_ST, kmaj(s0, 16384, ks), kmaj(stk, 16384, ks), idesc_bf16(128, 128), ks > 0);
#pragma unroll
        for (int ks = 0; ks < 6; ++ks)
            mma_bf16(tmem + TM_LF, mnmaj(r0, 12288, ks), kmaj(g0, 16384, ks),
                     idesc_bf16(128, 128, true, false), ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_RF, mnmaj(l0, 16384, ks), mnmaj(g0, 16384, ks),
                     idesc_bf16(128, 128, true, true), ks > 0);
        mma_commit(barM);
        mma_out = true;
        mma_out_ph = phM;
    }
    if (tid < C && tid < Lc)
        dbeta[(size_t)(row0 + tid) * H + h] += sDB[2 * tid] + sDB[2 * tid + 1];
    wait_mma();
    KDA_BWD_PHASE(4);

    // ---- per key channel c (TMEM lane c), tokens [32 hf, 32 hf + 32).  Group 2 is done:
    //      the stacked tile, S0 and G are free for fp32 tables [64 t][128 c].
    {
        float* gT = reinterpret_cast<float*>(sm + OFF_STK);   // cumulative log-gates g_t
        float* xT = reinterpret_cast<float*>(sm + OFF_S0);    // terms summed over r >= s
        float* yT = reinterpret_cast<float*>(sm + OFF_G);     // terms summed over j < s
        const int c = 32 * q4 + lane;
        const int t0 = 32 * hf;
        // column c of row t in a tile of 128-byte swizzled rows: (t >> 3) * 1024 + roff[t & 7]
        uint32_t roff[8];
        {
            const uint32_t cc = (uint32_t)((c & 63) >> 3), cb = (uint32_t)(c & 7) * 2u;
#pragma unroll
            for (int v = 0; v < 8; ++v) roff[v] = (uint32_t)v * 128u + (((cc ^ (uint32_t)v) & 7u) << 4) + cb;
        }
        const uint32_t at8 = (uint32_t)(c >> 6) * 8192u;    // 64-row tiles: alpha, q, k
        const uint8_t* sAl = sm + OFF_AL + at8;
        const uint8_t* sQ = sm + OFF_Q + at8;
        const uint8_t* sK = sm + OFF_K + at8;
        const uint8_t* sLt = sm + OFF_L + (uint32_t)(c >> 6) * 16384u;
        const uint8_t* sRt = sm + OFF_R + (uint32_t)(c >> 6) * 12288u;
        auto ld = [](const uint8_t* p) { return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p)); };
        // g_t = sum_{s <= t} log a_s (a = 1 past the chunk's tokens): each half its own
        // running sum; tokens 32..63 add the first half's total g_31 where they are read
        {
            float g = 0.0f;
#pragma unroll 1
            for (int u = 4 * hf; u < 4 * hf + 4; ++u) {
                float lg[8];
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const int t = 8 * u + v;
                    lg[v] = __logf(t < Lc ? clamp_gate(ld(sAl + (uint32_t)u * 1024u + roff[v])) : 1.0f);
                }
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    g += lg[v];
                    gT[(8 * u + v) * 128 + c] = g;
                }
            }
        }
        __syncthreads();
        KDA_BWD_PHASE(5);
        const float g31 = gT[31 * 128 + c];
        const float gadd = hf == 1 ? g31 : 0.0f;
        const float g15 = gT[15 * 128 + c], g47 = gT[47 * 128 + c] + g31, g63 = gT[63 * 128 + c] + g31;
        // token t of sub-chunk I (reference ref_I): lam_t = e^{g_t - g_ref} is the one
        // exponential; gamma_t = lam_t e^{g_ref}, rho^I_t = 1 / lam_t, eta_t = e^{g_63 - g_ref} / lam_t,
        // and for t < 32 rho^1_t = e^{g_47 - g_15} rho^0_t (every factor within e^+-80)
        const float gref_me = hf == 0 ? g15 : g47;   // (the half is the sub-chunk)
        const float Gref = __expf(gref_me), Eref = __expf(g63 - gref_me), P10 = __expf(g47 - g15);
        const float dgc = sDGC[c] + sDGC[128 + c];
        const size_t tstride = (size_t)H * DK;   // floats from one token's row to the next
        float* dq_c = dq + ((size_t)(row0 + t0) * H + h) * DK + c;
        float* dk_c = dk + ((size_t)(row0 + t0) * H + h) * DK + c;
        float sx = 0.f, sy = 0.f;
        // per block of 8 tokens: every load first, then the arithmetic, then the stores
        // (a table store followed by a load would otherwise order each token after the last)
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
            const int tb = t0 + 8 * blk;   // first token of this block (a multiple of 8)
            const bool sub0 = tb < 32;     // warp-uniform: sub-chunk 0 has the rho^0 operand
            const uint32_t rb = (uint32_t)(tb >> 3) * 1024u;
            float mdkt[8], dqt[8], dl[8], dlq[8], drf[8], dkh[8], dr0[8];
            tmem_ld8(tmem + tlane + TM_ST + tb, mdkt);
            tmem_ld8(tmem + tlane + TM_ST + 64 + tb, dqt);
            tmem_ld8(tmem + tlane + TM_LF + tb, dl);
            tmem_ld8(tmem + tlane + TM_LF + 64 + tb, dlq);
            tmem_ld8(tmem + tlane + TM_KH + tb, dkh);
            tmem_ld8(tmem + tlane + TM_RF + 32 + tb, drf);   // d(k*rho^1), rows 32 + t
            if (sub0) tmem_ld8(tmem + tlane + TM_RF + tb, dr0);   // d(k*rho^0), rows t < 32
            float gt[8], kv[8], qv[8], Lv[8], Lqv[8], R1v[8], R0v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t o = rb + roff[i];
                const bool live = tb + i < Lc;
                gt[i] = gT[(tb + i) * 128 + c] + gadd;
                kv[i] = live ? ld(sK + o) : 0.0f;
                qv[i] = live ? ld(sQ + o) : 0.0f;
                Lv[i] = ld(sLt + o);               // row t of [k*lam ; q*lam]
                Lqv[i] = ld(sLt + 8192u + o);      // row 64 + t
                R1v[i] = ld(sRt + 4096u + o);      // row 32 + t of [k*rho^0 ; k*rho^1]
                R0v[i] = sub0 ? ld(sRt + o) : 0.0f;
            }
            tmem_wait_ld();
            if (!sub0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) dr0[i] = 0.0f;
            }
            float x[8], y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float lam = __expf(gt[i] - gref_me), rl = __fdividef(1.0f, lam);
                const float gam = lam * Gref, eta = Eref * rl;
                const float rho0 = sub0 ? rl : 0.0f;
                const float rho1 = sub0 ? P10 * rl : rl;
                const float dkt = -mdkt[i];
                x[i] = (kv[i] * gam) * dkt + (qv[i] * gam) * dqt[i] + Lv[i] * dl[i] + Lqv[i] * dlq[i] -
                       R1v[i] * drf[i] - R0v[i] * dr0[i];
                y[i] = (kv[i] * eta) * dkh[i];
                dqt[i] = gam * dqt[i] + lam * dlq[i];
                mdkt[i] = gam * dkt + eta * dkh[i] + lam * dl[i] + rho1 * drf[i] + rho0 * dr0[i];   // dk
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                xT[(tb + i) * 128 + c] = x[i];
                yT[(tb + i) * 128 + c] = y[i];
                sx += x[i];
                sy += y[i];
                if (tb + i < Lc) {
                    const size_t o = (size_t)(8 * blk + i) * tstride;
                    dq_c[o] = dqt[i];
                    dk_c[o] = mdkt[i];
                }
            }
        }
        KDA_BWD_PHASE(6);
        // dlog a_s = sum_{r >= s} x_r + sum_{j < s} y_j + dgc, across the two token halves
        sTot[(hf * 2 + 0) * 128 + c] = sx;
        sTot[(hf * 2 + 1) * 128 + c] = sy;
        __syncthreads();
        float suf = hf == 0 ? sTot[(1 * 2 + 0) * 128 + c] : 0.0f;        // x of tokens 32..63
        float pre = (hf == 1 ? sTot[(0 * 2 + 1) * 128 + c] : 0.0f) + sy;  // y of tokens < t0 + 32
        float* da_c = dalpha + ((size_t)(row0 + t0) * H + h) * DK + c;
#pragma unroll 1
        for (int u = 3; u >= 0; --u) {
            float xs[8], ys[8], ar[8];
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int t = t0 + 8 * u + v;
                xs[v] = xT[t * 128 + c];
                ys[v] = yT[t * 128 + c];
                ar[v] = ld(sAl + (uint32_t)(t >> 3) * 1024u + roff[v]);
            }
#pragma unroll
            for (int v = 7; v >= 0; --v) {
                const int t = t0 + 8 * u + v;
                suf += xs[v];
                pre -= ys[v];   // y of tokens < t
                if (t < Lc) {
                    const float a = clamp_gate(ar[v]);
                    const bool pass = ar[v] >= kAlphaMin && ar[v] <= 1.0f;
                    da_c[(size_t)(8 * u + v) * tstride] = pass ? __fdividef(suf + pre + dgc, a) : 0.0f;
                }
            }
        }
    }

    if (!ok) atomicExch(sFlag, 1);
    __syncthreads();
    KDA_BWD_PHASE(7);
    if (*sFlag && issuer && mma_out) mbar_wait_ns(barM, mma_out_ph, kWaitNs);
    if (*sFlag && issuer) {   // the one phase of each load barrier
        mbar_wait_ns(barL, 0, kWaitNs);
        mbar_wait_ns(barL2, 0, kWaitNs);
    }
    __syncthreads();
    if (*sFlag && tid == 0) atomicExch(status, 1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace bwdtc

cudaError_t launch_chunk_tc_record(const void* q, const void* k, const void* v, const void* alpha,
                                   const void* beta, const float* S0, const int32_t* cu, int nseq,
                                   int64_t rows, int64_t T, int H, uint8_t* rec,
                                   bwdrec::Header* hdr, int64_t rec_chunks, int* status,
                                   cudaStream_t stream);

// Chunks the records are numbered over: dense, nseq * ceil(T / C); packed, at most
// ceil(T / C) + nseq (each sequence adds at most one partial chunk).
static int64_t backward_tc_chunks(bool packed, int64_t nseq, int64_t T) {
    return packed ? (T + bwdtc::C - 1) / bwdtc::C + nseq : nseq * ((T + bwdtc::C - 1) / bwdtc::C);
}

size_t backward_tc_workspace_bytes(bool packed, int64_t nseq, int64_t T, int H) {
    const int64_t nck = backward_tc_chunks(packed, nseq, T);
    return (size_t)nck * H * bwdrec::BYTES + (((size_t)nck * sizeof(bwdrec::Header) + 1023) & ~(size_t)1023);
}

// True where the tensor-core backward takes the call (bf16, d_k = d_v = 128, grid limits).
bool backward_tc_supported(bool bf16, int64_t nseq, int64_t T, int H, int DK, int DV, bool packed) {
    return bf16 && DK == 128 && DV == 128 && nseq <= 65535 && H <= 65535 &&
           backward_tc_chunks(packed, nseq, T) <= 0x7fffffffLL;
}

cudaError_t launch_backward_tc(const void* q, const void* k, const void* v, const void* alpha,
                               const void* beta, const float* S0, const void* dout,
                               const float* dSf, const int32_t* cu, int64_t nseq, int64_t T, int H,
                               float* dq, float* dk, float* dv, float* dalpha, float* dbeta,
                               float* dS0, void* workspace, int* status, cudaStream_t s) {
    const bool packed = cu != nullptr;
    const int64_t rows = packed ? T : nseq * T;
    const int64_t nck = backward_tc_chunks(packed, nseq, T);
    uint8_t* rec = static_cast<uint8_t*>(workspace);
    auto* hdr = reinterpret_cast<bwdrec::Header*>(rec + (size_t)nck * H * bwdrec::BYTES);
    if (rows == 0) return cudaSuccess;
    cudaError_t e = cudaMemsetAsync(hdr, 0, (size_t)nck * sizeof(bwdrec::Header), s);
    if (e != cudaSuccess) return e;
    e = launch_chunk_tc_record(q, k, v, alpha, beta, S0, cu, (int)nseq, rows, T, H, rec, hdr, nck,
                               status, s);
    if (e != cudaSuccess) return e;
    TcMaps m;   // m.v: dout; m.q, m.k, m.a: the inputs
    if (!make_tc_maps(&m, q, k, dout, alpha, nullptr, rows, H)) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(bwdtc::kda_bwd_dstate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bwdtc::ds::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    bwdtc::kda_bwd_dstate_kernel<<<dim3(1, H, (unsigned)nseq), bwdtc::NT + 32, bwdtc::ds::SMEM_BYTES, s>>>(
        m.v, static_cast<const __nv_bfloat16*>(beta), dSf, cu, T, H, rec, nck, dv, dbeta, dS0, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwdtc::kda_bwd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bwdtc::ck::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    bwdtc::kda_bwd_chunk_kernel<<<dim3((unsigned)nck, H), bwdtc::NT, bwdtc::ck::SMEM_BYTES, s>>>(
        m.v, m.a, m.q, m.k, static_cast<const __nv_bfloat16*>(beta), H, rec, hdr, dq, dk, dalpha,
        dbeta, status);
    return cudaGetLastError();
}

}  // namespace kda
