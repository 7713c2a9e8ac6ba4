// KDA chunked forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
// bf16 q, k, v, alpha, beta; fp32 state; d_k = d_v = 128; chunk C = 64.
//
// The worldcybernews article "Kimi K3 Open Model Surpasses Closed GPT and
// Anthropic Systems on Independent Benchmarks": paragraph 2 gives the state
// S (d_k x d_v), the delta-rule update with write strength beta and forget
// gate alpha in [e^-5, 1]; paragraph 3 processes the tokens of a chunk in
// parallel and carries the sequential state across chunks.  Per chunk, with
// start state S and a = clamp(alpha):
//
//   A[r,j] = beta_r sum_c k_rc k_jc D(r,j)_c  (j < r),  P[r,j] = sum_c q_rc k_jc D(r,j)_c  (j <= r)
//   D(r,j) = prod_{s=j+1..r} a_s,   Tinv = (I + A)^-1,   Tb = Tinv diag(beta)
//   W = Tb (k*gamma)                                   (gamma_r = prod_{s<=r} a_s)
//   U = -W S + Tb V = Tb (V - (k*gamma) S)
//   O = (q*gamma) S + P U
//   S <- Diag(gamma_C) S + (k*eta)^T U                  (eta_j = prod_{s>j} a_s)
//
// Only U and the state update are sequential from chunk to chunk; O is issued
// beside the state update.  The forward mode forms V - (k*gamma) S (its product
// issued beside [A/beta ; P], the difference taken while the solve runs) so that
// one M=64, K=64 MMA follows the solve; the summary mode, whose state is twice
// as wide, keeps the W form.  D(r,j) never appears as a ratio of long products
// (64 gates >= e^-5 reach e^-320, outside fp32/bf16): with 32-token
// sub-chunks I and the reference token ref_I = 32 I + 15,
//   D(r, j) = lam_r * rho^{I(r)}_j,  lam_r = e^{g_r - g_ref(I(r))},  rho^I_j = e^{g_ref(I) - g_j}
// (g the running log-gate), every factor within [e^-80, e^80] except right
// factors that underflow where the product itself is negligible.  All factors
// are running products of the clamped gates; nothing evaluates exp or log
// (except the optional transforms of the fused variant).  So
// [A/beta ; P] = [k*lam ; q*lam] [k*rho^0 ; k*rho^1]^T is one tcgen05 MMA group
// whose columns hold both sub-chunks' right operands.
//
// One CTA owns one (sequence, head) -- or one segment of it -- and walks its
// chunks in order: eight compute warps do the element-wise work, and one thread
// of a ninth (control) warp issues every TMA copy and MMA group at the barriers
// where the compute warps hand their operands over, so that MMA issue never
// stalls the compute warps.  Loads run about a chunk ahead: k and alpha once the
// gate phase has consumed them, q (double buffered) after the [A/beta ; P] MMA,
// v once U has consumed it.  O leaves through TMA stores from a staging tile.
// TMEM (512 columns): S fp32 [0,128), O [128,256), scratch accumulators
// [256,384), U [384,512) (first (k*gamma) S_start, then U).  Summary and dual
// modes: [M | N] fp32 [0,256); [256,512) holds in turn [A/beta ; P], the solve
// products, W, [U_M | U_N] and (dual) [Qg | O0].
//
// Long sequences with few (sequence, head) pairs are also split along time
// into segments (the prefix scan of paragraph 3, within one GPU).  Over a
// segment the state map is affine, S_end = M S_start + N with M (d_k x d_k) and
// N (d_k x d_v); per chunk M_c = Diag(gamma_C) - (k*eta)^T W and
// N_c = (k*eta)^T Tb V.  The same kernel in "summary" mode runs the chunk
// recurrence on [M | N] from [I | 0] without outputs (the maps of whole
// sequences); in "dual" mode it also forms that widened state's outputs
// [Qg | O0], whence o = O0 + Qg S_start.  The split forward runs every segment
// in the dual mode, chains S_{g+1} = M_g S_g + N_g in fp32 with a small scan
// kernel, and adds Qg S_g to the outputs with a last tensor-core kernel.
#include <cuda.h>

#include "kda_common.cuh"
#include "kda_sm100.cuh"
#include "kda_tc_maps.cuh"
#include "kda_bwd_record.cuh"

// Optional phase-boundary hook for profiling builds (no-op in the library).
#ifndef KDA_TC_PHASE
#define KDA_TC_PHASE(i)
#endif

namespace kda {
using namespace sm100;

namespace tc {

constexpr int C = 64;         // tokens per chunk
constexpr int DK = 128;       // key channels
constexpr int DV = 128;       // value channels
constexpr int NT = 256;       // compute threads (8 warps)
constexpr int NTHREADS = NT + 32;   // plus one control warp that issues every TMA copy and MMA
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait, then report a timeout

// shared-memory map (bytes from the 1024-aligned base)
constexpr uint32_t OFF_S = 0;            // S bf16 MN-major B [128 c][128 n], two atoms 16 KB apart;
                                         // a summary's [M | N] takes four atoms (64 KB, over the q tiles)
constexpr uint32_t OFF_Q = 32768;        // q tiles, two buffers of [64][128] (two [64][64] atoms each),
                                         // each becomes q*gamma in place (K-major A of the O MMA)
constexpr uint32_t OFF_K = 65536;        // k tile
constexpr uint32_t OFF_AL = 81920;       // alpha tile
constexpr uint32_t OFF_V = 98304;        // v tile: MN-major B, two 64-column atoms of [64][64]
constexpr uint32_t OFF_X = 114688;       // 72 KB work region, see below
constexpr uint32_t OFF_KT = OFF_X + 73728;   // k*gamma  MN-major B [64 j][128 c] (two [64][64] atoms)
constexpr uint32_t OFF_KH = OFF_KT + 16384;  // k*eta    MN-major A [64 j][128 c] (two [64][64] atoms)
constexpr uint32_t OFF_MISC = OFF_KH + 16384;
constexpr uint32_t MISC_PI = 0;          // float [8][128] octant gate products
constexpr uint32_t MISC_GC = 4096;       // float [128] gamma_C
constexpr uint32_t MISC_BETA = 4608;     // float [64]
constexpr uint32_t MISC_BAR = 4864;      // 6 x uint64 mbarriers: q, k+alpha (dual: k), v, MMA,
                                         // (k*gamma) S, alpha (dual mode)
constexpr uint32_t MISC_TMEM = 4912;     // uint32 TMEM base
constexpr uint32_t MISC_FLAG = 4916;     // int timeout seen
constexpr uint32_t SMEM_BYTES = OFF_MISC + 4928 + 1024;  // + alignment slack

// The dual mode (a segment's map [M | N] and both parts of its outputs, see the
// kernel) holds the 64 KB [M | N] copy and the q buffers at once: alpha and v take
// turns in one buffer (alpha is consumed at a chunk's start, v only at its barrier
// D), the work region ends at 64 KB, and the octant gate products live in its
// first 4 KB (free from the previous chunk's barrier E to this chunk's operand loop).
namespace dual {
constexpr uint32_t OFF_S = 0;            // [M | N] bf16, four [128][64] atoms
constexpr uint32_t OFF_Q = 65536;        // q, two buffers
constexpr uint32_t OFF_K = 98304;
constexpr uint32_t OFF_AV = 114688;      // alpha, then v
constexpr uint32_t OFF_X = 131072;       // 64 KB work region
constexpr uint32_t OFF_KT = 196608;
constexpr uint32_t OFF_KH = 212992;
constexpr uint32_t OFF_MISC = 229376 - 4096;   // the misc block without its first 4 KB (MISC_PI)
constexpr uint32_t X_PI = 0;             // float [8][128] octant gate products
constexpr uint32_t SMEM_BYTES = OFF_MISC + 4928 + 1024;
static_assert(SMEM_BYTES <= 232448, "dual-mode shared memory");
}  // namespace dual

// work region X, by phase
constexpr uint32_t X_L = 0;              // left rows [128][128]: k*lam rows 0..63, q*lam rows 64..127
constexpr uint32_t X_R = 32768;          // right rows [96][128]: k*rho^0 rows 0..31 (tokens 0..31),
                                         // k*rho^1 rows 32..95 (tokens 0..63); two 12 KB atoms
constexpr uint32_t X_P = 57344;          // P, K-major A [64 r][64 j]; lives until the O MMA
constexpr int AS = 68;                   // row stride (floats) of the fp32 A and Tinv tiles
constexpr uint32_t X_AM = 0;             // float A    [64][68]
constexpr uint32_t X_TM = 17408;         // float Tinv [64][68]
constexpr uint32_t X_XS = 34816;         // float scratch [32][36]
// fp32 K-major 128B-swizzled tiles (32 floats per row) for the tf32 MMAs of the 32 -> 64 step
constexpr uint32_t X_T0T = 40960;        // Tinv[0:32, 0:32]^T   [64 rows (32 used)][32]
constexpr uint32_t X_T1 = 49152;         // Tinv[32:64, 32:64]   [64 rows (32 used)][32]
constexpr uint32_t X_A10 = 45056;        // A[32:64, 0:32]       [32][32]: the rows 32..63 of the
                                         // T0^T tile, which its M=64 product reads but nobody uses
constexpr uint32_t X_TB = 40960;         // Tb, K-major A [64 r][64 m] (after the solve)
constexpr uint32_t X_WQ = 0;             // -W, K-major A [64][128] (two [64][64] atoms 8 KB apart)
constexpr uint32_t X_U = 16384;          // U, MN-major B [64 j][128 n] (two [64][64] atoms);
                                         // a summary's [U_M | U_N] takes four atoms

constexpr uint32_t TM_S = 0, TM_O = 128, TM_WK = 256, TM_U = 384;

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
    return row * 128u + (((chunk ^ row) & 7u) << 4);
}
// byte offset of fp32 element (r, k) in a K-major 128B-swizzled tile with 32 floats per row
__device__ __forceinline__ uint32_t f32_off(uint32_t r, uint32_t k) {
    return r * 128u + ((((k >> 2) ^ r) & 7u) << 4) + ((k & 3u) << 2);
}
__device__ __forceinline__ void unpack4_bf16(uint2 raw, float (&v)[4]) {
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
    v[0] = lo.x; v[1] = lo.y; v[2] = hi.x; v[3] = hi.y;
}
__device__ __forceinline__ void st4_bf16(uint8_t* p, const float (&v)[4]) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}

// 32 consecutive fp32 columns of this thread's TMEM lane, one wait for both loads
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(&v[0]));
    tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
    tmem_wait_ld();
}
// 64 consecutive fp32 columns of this thread's TMEM lane, one wait for all four loads
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
    tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(&v[0]));
    tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
    tmem_ld16(taddr + 32, *reinterpret_cast<float(*)[16]>(&v[32]));
    tmem_ld16(taddr + 48, *reinterpret_cast<float(*)[16]>(&v[48]));
    tmem_wait_ld();
}
__device__ __forceinline__ uint4 pack8(const float* v) {
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
}

// barrier among the eight compute warps only (the control warp is not held up)
__device__ __forceinline__ void sync_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// M=64 accumulator: row m lives in TMEM lane 32*(m/16) + m%16
// M=128 accumulator: row m lives in lane m.

// Time segments.  Sequence n's chunks are cut into `nseg` runs of
// ceil(chunks / nseg) chunks (the last ones may be shorter or empty); CTA z of
// a launch takes segment z % per_seq of the sequence of rank z / per_seq.
struct Segments {
    int nseg;             // segments per sequence (1: whole sequences)
    int per_seq;          // segment CTAs per sequence in this launch
    const float* start;   // forward with nseg > 1: start states [nseq * nseg, H, DK, DV]
                          // (a form no entry point launches now: the split forward takes
                          // the dual mode and adds the start states' share afterwards)
    float* maps;          // summary: [M | N] fp32 [nseq * per_seq, H, DK, DK + DV]
    // state slots (whole sequences only): sequence n reads S0 and writes S_final at
    // slot slots[n] of a pool of num_slots states; a slot outside [0, num_slots)
    // starts from zero and writes no state.  Null: slot n.
    const int32_t* slots;
    int num_slots;
    // dual mode: the per-token map rows Qg [rows, H, DK] bf16 (see the kernel)
    __nv_bfloat16* qg = nullptr;
    // record mode (the backward's first pass): per-(chunk, head) records and per-chunk
    // headers, chunks numbered across sequences in order
    uint8_t* rec = nullptr;
    bwdrec::Header* hdr = nullptr;
    int64_t rec_chunks = 0;   // chunks the records hold (a malformed packed table is cut there)
};

// One TMA stream's bookkeeping: the parity a thread's next wait on it expects,
// and (control thread) how many loads were issued on it.
struct LoadTrack {
    uint32_t ph = 0, issued = 0;
};

// kCtaStatus = false: a timed-out wait sets the shared word *status to 1.
// kCtaStatus = true:  every CTA writes its own word status[n * H + h] (0 or 1).
// kSummary = true: the segment-map mode described at the top (q and out unused).
// kFused = true: alpha and beta arrive as logits (alpha = 1/(1+e^x), beta =
// sigmoid(x)) and q, k unnormalised (L2-normalised per token and head here).
// kRecord = true: the forward recurrence without outputs; every chunk's start state,
// operand tiles, T, V - (k*gamma) S, U and gamma_C go to the backward's record of
// (chunk, head) (kda_bwd_record.cuh), byte for byte as they sit in shared memory.
// kDual = true (with kSummary): the summary recurrence on [M | N] from [I | 0] that also
// forms the chunk outputs of that 256-wide state, [Qg | O0] = (q*gamma) [M | N] + P
// [U_M | U_N]: O0 is the segment's output from a zero start state (written to out)
// and Qg (written to seg.qg) the rows that carry its true start state S_g into it,
// o = O0 + Qg S_g (the state map is affine, so the output is too).  One pass over a
// segment then gives both its map and everything its outputs need but S_g.
template <bool kCtaStatus, bool kSummary, bool kFused, bool kRecord = false, bool kDual = false>
__global__ void __launch_bounds__(NTHREADS, 1)
kda_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmG,
                    const __nv_bfloat16* __restrict__ beta, const float* S0,
                    const int32_t* __restrict__ cu_seqlens, __nv_bfloat16* __restrict__ out,
                    float* S_final, int64_t T, int H, int* status, const Segments seg) {
    extern __shared__ uint8_t smem_raw[];
    // the 1024-aligned base as an offset into the shared array, so that the compiler
    // keeps every access below a shared-memory one (measured: 1.060 -> 0.975 ms on the
    // 4096-token batch); the fused variant keeps the generic pointer, with which its
    // register allocation spills less (1.62 against 1.83 ms)
    uint8_t* sm = kFused ? reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                      ~static_cast<uintptr_t>(1023))
                         : smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    static_assert(!kDual || (kSummary && !kRecord), "the dual mode is a summary mode");
    constexpr bool kQ = !kSummary || kDual;   // q is read and outputs are formed
    constexpr uint32_t oMisc = kDual ? dual::OFF_MISC : OFF_MISC;
    uint8_t* sS = sm + (kDual ? dual::OFF_S : OFF_S);
    uint8_t* sQ = sm + (kDual ? dual::OFF_Q : OFF_Q);
    uint8_t* sK = sm + (kDual ? dual::OFF_K : OFF_K);
    uint8_t* sAl = sm + (kDual ? dual::OFF_AV : OFF_AL);
    uint8_t* sV = sm + (kDual ? dual::OFF_AV : OFF_V);
    uint8_t* sX = sm + (kDual ? dual::OFF_X : OFF_X);
    uint8_t* sKT = sm + (kDual ? dual::OFF_KT : OFF_KT);
    uint8_t* sKH = sm + (kDual ? dual::OFF_KH : OFF_KH);
    float* sPi = reinterpret_cast<float*>(kDual ? sX + dual::X_PI : sm + OFF_MISC + MISC_PI);
    float* sGC = reinterpret_cast<float*>(sm + oMisc + MISC_GC);
    float* sBeta = reinterpret_cast<float*>(sm + oMisc + MISC_BETA);
    uint64_t* barQ = reinterpret_cast<uint64_t*>(sm + oMisc + MISC_BAR);
    uint64_t* barKA = barQ + 1;
    uint64_t* barV = barQ + 2;
    uint64_t* barM = barQ + 3;
    uint64_t* barZ = barQ + 4;   // (k*gamma) S_start, forward mode
    uint64_t* barAl = barQ + 5;  // alpha, dual mode
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + oMisc + MISC_TMEM);
    int* sFlag = reinterpret_cast<int*>(sm + oMisc + MISC_FLAG);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool compute = warp < NT / 32;   // warps 0-7; warp 8 is the control warp
    const bool ctl = warp == NT / 32 && lane == 0;   // the thread that issues copies and MMAs
    const int q4 = warp & 3;            // TMEM lane quarter this warp may touch
    const int hf = warp >> 2;           // which half of the columns this warp handles
    const int h = blockIdx.y;
    const int per_seq = seg.per_seq, gseg = (int)blockIdx.z % per_seq;
    __shared__ int s_seq;
    __shared__ int64_t s_cbase;
    if (threadIdx.x < 32) {
        const int sq = longest_first_seq(cu_seqlens, (int)gridDim.z / per_seq,
                                         (int)blockIdx.z / per_seq, T);
        const int64_t cb = kRecord ? chunks_before(cu_seqlens, sq, T, C) : 0;
        if (threadIdx.x == 0) { s_seq = sq; s_cbase = cb; }
    }
    __syncthreads();
    const int n = s_seq;
    // this CTA's record of chunk i (record mode)
    auto rec_of = [&](int i) {
        return seg.rec + ((size_t)(s_cbase + i) * H + h) * bwdrec::BYTES;
    };
    int64_t bos, len;
    seq_range(cu_seqlens, n, T, bos, len);
    if (seg.nseg > 1) {   // this CTA's segment of the sequence
        const int64_t nch = (len + C - 1) / C, cps = (nch + seg.nseg - 1) / seg.nseg;
        const int64_t c0 = min((int64_t)gseg * cps, nch), c1 = min((int64_t)(gseg + 1) * cps, nch);
        const int64_t t0 = min(c0 * C, len), t1 = min(c1 * C, len);
        bos += t0;
        len = t1 - t0;
    }
    int nchunks = (int)((len + C - 1) / C);
    if (kRecord && s_cbase + nchunks > seg.rec_chunks)
        nchunks = (int)max((int64_t)0, seg.rec_chunks - s_cbase);
    const bool last_seg = gseg == seg.nseg - 1;
    const int slot = seg.slots ? seg.slots[n] : n;
    const bool slot_ok = !seg.slots || (slot >= 0 && slot < seg.num_slots);

    if (tid == 0) {
        mbar_init(barQ, 1);
        mbar_init(barKA, 1);
        mbar_init(barV, 1);
        mbar_init(barM, 1);
        mbar_init(barZ, 1);
        mbar_init(barAl, 1);
        mbar_fence_init();
        *sFlag = 0;
    }
    if (warp == 0) tmem_alloc(sTmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    KDA_TC_PHASE(30);
    const uint32_t tmem = *sTmem;
    const uint32_t tlane = (uint32_t)(32 * q4) << 16;

    // ---- initial state: TMEM S (fp32) and its bf16 copy (MN-major B operand)
    if (!compute) {
    } else if constexpr (kSummary) {
        // [M | N] = [I | 0]; this warp writes row c, columns 128 hf .. 128 hf + 127
        const int c = 32 * q4 + lane;
#pragma unroll
        for (int blk = 0; blk < 8; ++blk) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = (128 * hf + 16 * blk + i == c) ? 1.0f : 0.0f;
            tmem_st16(tmem + tlane + TM_S + 128 * hf + 16 * blk, v);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
                *reinterpret_cast<uint4*>(sS + (2 * hf + (blk >> 2)) * 16384 +
                                          swz(c, 2 * (blk & 3) + ch)) = pack8(&v[8 * ch]);
        }
        tmem_wait_st();
    } else {
        const int c = 32 * q4 + lane;
        const float* base = seg.nseg > 1
                                ? seg.start + (((size_t)n * seg.nseg + gseg) * H + h) * DK * DV
                                : (S0 && slot_ok ? S0 + ((size_t)slot * H + h) * DK * DV : nullptr);
        const float* src = base ? base + (size_t)c * DV + 64 * hf : nullptr;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
                float4 f = src ? *reinterpret_cast<const float4*>(src + 16 * blk + i)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                v[i] = f.x; v[i + 1] = f.y; v[i + 2] = f.z; v[i + 3] = f.w;
            }
            tmem_st16(tmem + tlane + TM_S + 64 * hf + 16 * blk, v);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
                *reinterpret_cast<uint4*>(sS + hf * 16384 + swz(c, 2 * blk + ch)) = pack8(&v[8 * ch]);
        }
        tmem_wait_st();
    }

    auto issue_q = [&](int64_t row0, int buf) {
        mbar_arrive_expect_tx(barQ, 16384);
#pragma unroll
        for (int a = 0; a < 2; ++a)
            tma_load_2d(sQ + buf * 16384 + a * 8192, &tmQ, barQ, h * DK + 64 * a, (int)row0);
    };
    auto issue_ka = [&](int64_t row0) {   // k and (but in the dual mode) alpha
        mbar_arrive_expect_tx(barKA, kDual ? 16384 : 2 * 16384);
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            tma_load_2d(sK + a * 8192, &tmK, barKA, h * DK + 64 * a, (int)row0);
            if (!kDual) tma_load_2d(sAl + a * 8192, &tmA, barKA, h * DK + 64 * a, (int)row0);
        }
    };
    auto issue_al = [&](int64_t row0) {   // dual mode: alpha, into the buffer v leaves
        mbar_arrive_expect_tx(barAl, 16384);
#pragma unroll
        for (int a = 0; a < 2; ++a)
            tma_load_2d(sAl + a * 8192, &tmA, barAl, h * DK + 64 * a, (int)row0);
    };
    auto issue_v = [&](int64_t row0) {
        mbar_arrive_expect_tx(barV, 16384);
#pragma unroll
        for (int a = 0; a < 2; ++a)
            tma_load_2d(sV + a * 8192, &tmV, barV, h * DV + 64 * a, (int)row0);
    };

    bool ok = true;   // this thread has seen every wait complete
    // asynchronous work that a timed-out wait may leave in flight, drained before exit
    LoadTrack tq, tka, tv, tal;
    uint32_t phM = 0, mma_out_ph = 0, phZ = 0, z_out_ph = 0;
    bool mma_out = false;   // (control thread) an MMA group committed and not yet waited for
    bool z_out = false;     // (control thread) the same for the (k*gamma) S group
    auto wait_load = [&](uint64_t* bar, LoadTrack& t) {
        if (ok && !mbar_wait_ns(bar, t.ph, kWaitNs)) ok = false;
        t.ph ^= 1u;
    };
    auto issued = [&](LoadTrack& t) { ++t.issued; };
    auto commit_mma = [&]() {   // control thread, after issuing an MMA group
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
    auto commit_z = [&]() {
        mma_commit(barZ);
        z_out = true;
        z_out_ph = phZ;
    };
    auto wait_z = [&]() {
        if (ok) {
            if (mbar_wait_ns(barZ, phZ, kWaitNs)) z_out = false;
            else ok = false;
        }
        phZ ^= 1u;
        tc_fence_after();
    };

    // The state update (and O) of a chunk is waited for, and its results taken out
    // of TMEM, only inside the next chunk's gate phase: nothing before the next
    // chunk's U MMA needs them.  S goes to its bf16 copy, O to the output rows.
    // A full chunk's O is staged in the q buffer the next q load will use (row-major,
    // 128-byte swizzled, the TMA box layout) and written by one TMA store; a
    // partial last chunk is stored row by row.  The dual mode's [Qg | O0] (an M=64
    // accumulator, N=256; warps of column half 0 hold Qg, half 1 O0) is staged the same
    // way, O0 in that q buffer and Qg in the alpha / v buffer (alpha is read, v not yet
    // loaded): both are free from here until the control thread's stores at barrier A.
    auto finish_prev = [&](int64_t prow0, int pLc, uint8_t* stage) {
        wait_mma();
        const int c = 32 * q4 + lane;
        if constexpr (kDual && !kFused) {   // (32-column pieces: fewer live registers)
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                float v[32];
                tmem_ld32(tmem + tlane + TM_S + 128 * hf + 32 * p, v);
#pragma unroll
                for (int ch = 0; ch < 4; ++ch)
                    *reinterpret_cast<uint4*>(sS + (2 * hf + (p >> 1)) * 16384 + swz(c, 4 * (p & 1) + ch)) =
                        pack8(&v[8 * ch]);
            }
        } else if constexpr (kSummary) {
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float v[64];
                tmem_ld64(tmem + tlane + TM_S + 128 * hf + 64 * p, v);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4*>(sS + (2 * hf + p) * 16384 + swz(c, ch)) = pack8(&v[8 * ch]);
            }
        }
        if constexpr (kSummary) {
            if constexpr (kDual) {
                const int r = 16 * q4 + lane;
                if (pLc == C) {
                    uint8_t* stg = (hf == 0 ? sAl : stage) + r * 128;   // row r of both atoms
                    const uint32_t rx = (uint32_t)(r & 7);
#pragma unroll 1
                    for (int p = 0; p < 4; ++p) {   // (32-column pieces: fewer live registers)
                        float v[32];
                        tmem_ld32(tmem + tlane + TM_WK + 128 * hf + 32 * p, v);
                        if (lane < 16) {
#pragma unroll
                            for (int ch = 0; ch < 4; ++ch)
                                *reinterpret_cast<uint4*>(stg + (p >> 1) * 8192 + (((4 * (p & 1) + ch) ^ rx) << 4)) =
                                    pack8(&v[8 * ch]);
                        }
                    }
                } else {
                    uint4* dst = reinterpret_cast<uint4*>((hf == 0 ? seg.qg : out) + ((size_t)(prow0 + r) * H + h) * DK);
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        float v[32];
                        tmem_ld32(tmem + tlane + TM_WK + 128 * hf + 32 * p, v);
                        if (lane < 16 && r < pLc) {
#pragma unroll
                            for (int ch = 0; ch < 4; ++ch) dst[4 * p + ch] = pack8(&v[8 * ch]);
                        }
                    }
                }
            }
        } else {
            float v[64];
            tmem_ld64(tmem + tlane + TM_S + 64 * hf, v);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4*>(sS + hf * 16384 + swz(c, ch)) = pack8(&v[8 * ch]);
            if constexpr (kRecord) return;   // no outputs
            tmem_ld64(tmem + tlane + TM_O + 64 * hf, v);
            const int r = 16 * q4 + lane;
            if (pLc == C) {
                if (lane < 16) {
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        *reinterpret_cast<uint4*>(stage + hf * 8192 + swz(r, ch)) = pack8(&v[8 * ch]);
                }
            } else if (lane < 16 && r < pLc) {
                uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)(prow0 + r) * H + h) * DV + 64 * hf);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) dst[ch] = pack8(&v[8 * ch]);
            }
        }
    };
    auto store_o = [&](uint8_t* stage, int64_t prow0) {   // control thread, after a barrier
#pragma unroll
        for (int a = 0; a < 2; ++a) tma_store_2d(&tmO, stage + a * 8192, h * DV + 64 * a, (int)prow0);
        bulk_commit_group();
    };
    auto store_dual = [&](uint8_t* stage, int64_t prow0) {   // dual mode: O0 and Qg of a full chunk
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            tma_store_2d(&tmO, stage + a * 8192, h * DV + 64 * a, (int)prow0);
            tma_store_2d(&tmG, sAl + a * 8192, h * DK + 64 * a, (int)prow0);
        }
        bulk_commit_group();
    };

    if (nchunks > 0 && ctl) {
        if (kQ) {
            issue_q(bos, 0);
            issued(tq);
        }
        issue_ka(bos);
        issued(tka);
        if (kDual) {   // v follows once the first chunk's gate phase has read alpha
            issue_al(bos);
            issued(tal);
        } else {
            issue_v(bos);
            issued(tv);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // beta of the next chunk is loaded one chunk ahead, into a register
    constexpr bool fused = kFused;
    auto load_beta = [&](int64_t token) {   // token index in the segment, < len
        const float x = __bfloat162float(beta[(size_t)(bos + token) * H + h]);
        return fused ? sigmoid_f(x) : x;
    };
    float beta_next = 0.0f;
    if (tid < C && tid < len) beta_next = load_beta(tid);

    bool broke = false;
    if (compute)
    for (int chunk = 0; chunk < nchunks; ++chunk) {
        const int64_t row0 = bos + (int64_t)chunk * C;
        const int Lc = (int)((len - (int64_t)chunk * C) < C ? (len - (int64_t)chunk * C) : C);
        uint8_t* sQc = sQ + (chunk & 1) * 16384;
        if (tid < C) sBeta[tid] = beta_next;
        wait_load(barKA, tka);
        if (kDual) wait_load(barAl, tal);
        if (kQ) wait_load(barQ, tq);
        KDA_TC_PHASE(0);

        // ================= gate products and bf16 operands (all threads)
        {
            // thread = (channels c0..c0+3) x (8-token octant O).  Quarter Q = O/2 holds 16
            // tokens, sub-chunk I = Q/2 holds 32; the reference token of I is ref_I = 32I + 15.
            // With phi / psi the in-quarter forward (inclusive) / backward (exclusive) gate
            // products and pi_Q the quarter product:
            //   left  lam_t   = e^{g_t - g_ref}  = phi_t * (Q even ? 1/pi_Q : 1)
            //   right rho^I_j = e^{g_ref - g_j}  = psi_j * c_I(Q(j))
            //   c_0 = {1, 1/pi_1},  c_1 = {pi_1 pi_2, pi_2, 1, 1/pi_3}
            // so that lam_r rho^I_j = prod_{s=j+1..r} a_s for j <= r, every factor within
            // [e^-80, e^80] except right factors that underflow where the product is negligible.
            // In-quarter products come from in-octant ones phi8, psi8 and the octant products
            // pi8: phi = phi8 * (O odd ? pi8_{O-1} : 1), psi = psi8 * (O even ? pi8_{O+1} : 1);
            // those octant factors are folded into the per-thread scales below.
            // Every tile touched here is row-major with 128-byte swizzled rows; a warp covers
            // one token row of all 128 channels (8 bytes per thread).
            const int cq = tid & 31, O = tid >> 5, Q = O >> 1, c0 = 4 * cq;
            const uint32_t chk = (uint32_t)((c0 & 63) >> 3), inner = (uint32_t)((c0 & 7) << 1);
            const uint32_t a64 = (uint32_t)(c0 >> 6);
            float phi[8][4], psi[8][4];   // psi holds the clamped gates until the backward pass
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 8 * O + i;
                const uint32_t off = a64 * 8192u + (uint32_t)r * 128u + (((chk ^ (uint32_t)r) & 7u) << 4) + inner;
                float a[4];
                unpack4_bf16(*reinterpret_cast<const uint2*>(sAl + off), a);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    psi[i][c] = r < Lc ? clamp_gate(fused ? gate_from_logit(a[c]) : a[c]) : 1.0f;
            }
            {
                float p[4] = {1.f, 1.f, 1.f, 1.f}, b[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int c = 0; c < 4; ++c) { p[c] *= psi[i][c]; phi[i][c] = p[c]; }
#pragma unroll
                for (int i = 7; i >= 0; --i)
#pragma unroll
                    for (int c = 0; c < 4; ++c) { const float a = psi[i][c]; psi[i][c] = b[c]; b[c] *= a; }
                *reinterpret_cast<float4*>(&sPi[O * DK + c0]) = make_float4(p[0], p[1], p[2], p[3]);
            }
            KDA_TC_PHASE(13);
            sync_compute();
            KDA_TC_PHASE(14);
            // the previous chunk's state update and O (their operands KH, U, P and the
            // q buffer are overwritten from here on)
            if (chunk > 0) finish_prev(row0 - C, C, sQ + ((chunk + 1) & 1) * 16384);
            KDA_TC_PHASE(15);
            // per-thread scales: quarter products, gamma before / eta after this quarter
            float dlf[4], bf[4], r0g[4], r1g[4], ag[4];
            {
                float pq[4][4];   // [quarter][channel]
#pragma unroll
                for (int M = 0; M < 4; ++M) {
                    const float4 u = *reinterpret_cast<const float4*>(&sPi[(2 * M) * DK + c0]);
                    const float4 v = *reinterpret_cast<const float4*>(&sPi[(2 * M + 1) * DK + c0]);
                    pq[M][0] = u.x * v.x; pq[M][1] = u.y * v.y; pq[M][2] = u.z * v.z; pq[M][3] = u.w * v.w;
                }
                // the partner octant of this quarter: phi8 -> phi (O odd), psi8 -> psi (O even)
                const float4 po = *reinterpret_cast<const float4*>(&sPi[(O ^ 1) * DK + c0]);
                const float pov[4] = {po.x, po.y, po.z, po.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float bef = 1.f, aft = 1.f, own = 1.f;
#pragma unroll
                    for (int M = 0; M < 4; ++M) {
                        if (M < Q) bef *= pq[M][c];
                        if (M > Q) aft *= pq[M][c];
                        if (M == Q) own = pq[M][c];
                    }
                    if (O == 0) sGC[c0 + c] = pq[0][c] * pq[1][c] * pq[2][c] * pq[3][c];
                    if (kRecord && O == 0)
                        reinterpret_cast<float*>(rec_of(chunk) + bwdrec::GC)[c0 + c] = sGC[c0 + c];
                    const float fO = (O & 1) ? pov[c] : 1.0f;
                    const float gO = (O & 1) ? 1.0f : pov[c];
                    const float dl = (Q & 1) ? 1.0f : __frcp_rn(own);
                    const float r0 = Q == 1 ? __frcp_rn(own) : 1.0f;
                    const float r1 = Q == 0 ? pq[1][c] * pq[2][c]
                                            : (Q == 1 ? pq[2][c] : (Q == 2 ? 1.0f : __frcp_rn(own)));
                    dlf[c] = dl * fO;
                    bf[c] = bef * fO;
                    r0g[c] = r0 * gO;
                    r1g[c] = r1 * gO;
                    ag[c] = aft * gO;
                }
            }
            // fused inputs: the L2 norms of this warp's eight k (and q) rows (a warp holds all
            // 128 channels of its rows, four per lane); the operand loop below scales the rows
            // as it reads them, so nothing is written back
            float kinv[8], qinv[8];
            if constexpr (kFused) {
                float sk[8], sq[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 8 * O + i;
                    const uint32_t in_off = a64 * 8192u + (uint32_t)r * 128u + (((chk ^ (uint32_t)r) & 7u) << 4) + inner;
                    float k[4], q[4] = {0.f, 0.f, 0.f, 0.f};
                    unpack4_bf16(*reinterpret_cast<const uint2*>(sK + in_off), k);
                    if (kQ) unpack4_bf16(*reinterpret_cast<const uint2*>(sQc + in_off), q);
                    sk[i] = k[0] * k[0] + k[1] * k[1] + k[2] * k[2] + k[3] * k[3];
                    sq[i] = q[0] * q[0] + q[1] * q[1] + q[2] * q[2] + q[3] * q[3];
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], o);
                        if (kQ) sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], o);
                    }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    kinv[i] = rsqrtf(fmaxf(sk[i], 1e-12f));
                    qinv[i] = rsqrtf(fmaxf(sq[i], 1e-12f));
                }
            }
            // each row's k (and q) is read before the previous row's stores: q*gamma is
            // written in place, so a load placed after a store could not be moved above it
            auto in_off_of = [&](int r) {
                return a64 * 8192u + (uint32_t)r * 128u + (((chk ^ (uint32_t)r) & 7u) << 4) + inner;
            };
            // dual mode: the gate products sit where the operand tiles go
            if constexpr (kDual) sync_compute();
            uint2 kn = *reinterpret_cast<const uint2*>(sK + in_off_of(8 * O));
            uint2 qn = !kQ ? make_uint2(0u, 0u) : *reinterpret_cast<const uint2*>(sQc + in_off_of(8 * O));
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 8 * O + i;
                const uint32_t sw = (uint32_t)r * 128u + (((chk ^ (uint32_t)r) & 7u) << 4) + inner;
                const uint32_t in_off = a64 * 8192u + sw;    // 64-row tiles: q, k, KT, KH
                float k[4], q[4] = {0.f, 0.f, 0.f, 0.f};
                unpack4_bf16(kn, k);
                if (kQ) unpack4_bf16(qn, q);
                if constexpr (kFused) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) { k[c] *= kinv[i]; q[c] *= qinv[i]; }
                }
                if (i < 7) {
                    kn = *reinterpret_cast<const uint2*>(sK + in_off_of(r + 1));
                    if (kQ) qn = *reinterpret_cast<const uint2*>(sQc + in_off_of(r + 1));
                }
                if (r >= Lc) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) { k[c] = 0.0f; q[c] = 0.0f; }
                }
                float kp[4], qp[4], ks[4], w[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    kp[c] = k[c] * phi[i][c];
                    qp[c] = q[c] * phi[i][c];
                    ks[c] = k[c] * psi[i][c];
                }
                uint8_t* lrow = sX + X_L + a64 * 16384u + sw;             // 128-row atoms
                uint8_t* rrow = sX + X_R + a64 * 12288u + sw;             // 96-row atoms
#pragma unroll
                for (int c = 0; c < 4; ++c) w[c] = kp[c] * dlf[c];
                st4_bf16(lrow, w);                                        // k*lam, row r
                if (kQ) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) w[c] = qp[c] * dlf[c];
                    st4_bf16(lrow + 64 * 128, w);                         // q*lam, row 64 + r
#pragma unroll
                    for (int c = 0; c < 4; ++c) w[c] = qp[c] * bf[c];
                    st4_bf16(sQc + in_off, w);                            // q*gamma in place
                }
                if (O < 4) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) w[c] = ks[c] * r0g[c];
                    st4_bf16(rrow, w);                                    // k*rho^0, row r < 32
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) w[c] = ks[c] * r1g[c];
                st4_bf16(rrow + 32 * 128, w);                             // k*rho^1, row 32 + r
#pragma unroll
                for (int c = 0; c < 4; ++c) w[c] = kp[c] * bf[c];
                st4_bf16(sKT + in_off, w);                                // k*gamma
#pragma unroll
                for (int c = 0; c < 4; ++c) w[c] = ks[c] * ag[c];
                st4_bf16(sKH + in_off, w);                                // k*eta
            }
            KDA_TC_PHASE(16);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        KDA_TC_PHASE(1);
        // ================= [A/beta ; P] = [k*lam ; q*lam] [k*rho^0 ; k*rho^1]^T   (M=128, N=96, K=128)
        //   rows 0..63 are A/beta rows r, rows 64..127 are P rows r.  Columns [0, 32) hold
        //   rho^0 (j < 32, valid for r < 32), columns [32, 96) hold rho^1 (j < 64, valid for r >= 32).
        // meanwhile: S (summary: [M | N]) <- Diag(gamma_C) S in TMEM -- the MMAs read the
        // bf16 copy, and only the state update, hand-offs later, accumulates onto S
        {
            const int c = 32 * q4 + lane;
            const float g = sGC[c];
            constexpr int ncol = kSummary ? 128 : 64;   // this thread's columns
#pragma unroll
            for (int blk = 0; blk < ncol / 16; ++blk) {
                float w[16];
                tmem_ld16(tmem + tlane + TM_S + ncol * hf + 16 * blk, w);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) w[i] *= g;
                tmem_st16(tmem + tlane + TM_S + ncol * hf + 16 * blk, w);
            }
            tmem_wait_st();
        }
        wait_mma();

        KDA_TC_PHASE(2);
        // ================= A (fp32, times beta_r, j < r) and P (bf16 K-major A operand, j <= r)
        {
            // lane = row R of the accumulator: R < 64 is A row r = R, R >= 64 is P row r = R - 64;
            // this warp's column half covers j in [32 hf, 32 hf + 32)
            const int R = 32 * q4 + lane, r = R & 63, j0 = 32 * hf;
            const bool lower = (q4 & 1) == 0;          // r < 32: group 1 columns
            const bool zero = lower && hf == 1;        // j >= 32 > r: all zero
            float v[32];
            if (!zero && (q4 < 2 || kQ)) {
                const uint32_t col = lower ? 0u : 32u + 32u * hf;
                tmem_ld16(tmem + tlane + TM_WK + col, *reinterpret_cast<float(*)[16]>(&v[0]));
                tmem_ld16(tmem + tlane + TM_WK + col + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.0f;
            }
            if (q4 < 2) {
                float* Am = reinterpret_cast<float*>(sX + X_AM);
                const float b = sBeta[r];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float4 f;
                    f.x = (j0 + i + 0 < r) ? b * v[i + 0] : 0.0f;
                    f.y = (j0 + i + 1 < r) ? b * v[i + 1] : 0.0f;
                    f.z = (j0 + i + 2 < r) ? b * v[i + 2] : 0.0f;
                    f.w = (j0 + i + 3 < r) ? b * v[i + 3] : 0.0f;
                    *reinterpret_cast<float4*>(&Am[r * AS + j0 + i]) = f;
                }
            } else if (kQ) {
                uint8_t* sP = sX + X_P;
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    float w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) w[i] = (j0 + 8 * c8 + i <= r) ? v[8 * c8 + i] : 0.0f;
                    *reinterpret_cast<uint4*>(sP + swz(r, (j0 >> 3) + c8)) = pack8(w);
                }
            }
        }
        // no proxy fence here: A is read by the CUDA cores, and P by an MMA only after the
        // fenced hand-off that precedes the tf32 solve products
        tc_fence_before();
        sync_compute();
        KDA_TC_PHASE(3);
        // ================= Tinv = (I + A)^-1 by doubling: 16x16 blocks, then 32, then 64
        //   inv([[X, 0], [Y, Z]]) = [[X^-1, 0], [-Z^-1 Y X^-1, Z^-1]]
        {
            const float* Am = reinterpret_cast<const float*>(sX + X_AM);
            float* Tm = reinterpret_cast<float*>(sX + X_TM);
            float* Xs = reinterpret_cast<float*>(sX + X_XS);
            if (warp < 4) {
                // diagonal 16x16 blocks by forward substitution: warp I, lane m < 16 owns column m
                const int I = warp, m = lane & 15, o = 16 * I;
                float col[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float arow[16];
#pragma unroll
                    for (int jj = 0; jj < 16; jj += 4)
                        if (jj < r) *reinterpret_cast<float4*>(&arow[jj]) =
                            *reinterpret_cast<const float4*>(&Am[(o + r) * AS + o + jj]);
                    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
#pragma unroll
                    for (int jj = 0; jj < r; ++jj) {
                        if ((jj & 3) == 0) s0 = fmaf(arow[jj], col[jj], s0);
                        else if ((jj & 3) == 1) s1 = fmaf(arow[jj], col[jj], s1);
                        else if ((jj & 3) == 2) s2 = fmaf(arow[jj], col[jj], s2);
                        else s3 = fmaf(arow[jj], col[jj], s3);
                    }
                    col[r] = r < m ? 0.0f : (r == m ? 1.0f : -((s0 + s1) + (s2 + s3)));
                }
                if (lane < 16) {
#pragma unroll
                    for (int r = 0; r < 16; ++r) Tm[(o + r) * AS + o + m] = col[r];
                }
            } else {
                // zeros above the diagonal blocks that the doubling steps read
                const int t = tid - 128;                       // 0..127
                const int r = t >> 2, cq = (t & 3) * 4;        // rows 0..31, 4 columns each
                const int rb = r < 16 ? r : 16 + r;            // rows 0-15 and 32-47
                const int cb = r < 16 ? 16 + cq : 48 + cq;     // columns 16-31 and 48-63
                *reinterpret_cast<float4*>(&Tm[rb * AS + cb]) = make_float4(0.f, 0.f, 0.f, 0.f);
                const int r2 = t >> 2;                         // rows 0..31, columns 32..63
#pragma unroll
                for (int c4 = 0; c4 < 2; ++c4)
                    *reinterpret_cast<float4*>(&Tm[r2 * AS + 32 + 16 * c4 + cq]) =
                        make_float4(0.f, 0.f, 0.f, 0.f);
                if constexpr (!kSummary) {
                    // V - (k*gamma) S_start, written over the v tile (the MN-major B operand of
                    // the U MMA).  (k*gamma) S_start is an M=64 accumulator in U's columns:
                    // row j = 16 q4 + lane for lane < 16.
                    wait_z();
                    KDA_TC_PHASE(17);
                    wait_load(barV, tv);
                    KDA_TC_PHASE(18);
                    const int j = 16 * q4 + lane;
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        float z[64];
                        tmem_ld64(tmem + tlane + TM_U + 64 * a, z);
                        if (lane < 16) {
                            // each 16-byte piece is read before the previous one is written back
                            uint4 nxt = *reinterpret_cast<const uint4*>(sV + a * 8192 + swz(j, 0));
#pragma unroll
                            for (int ch = 0; ch < 8; ++ch) {
                                const uint4 raw = nxt;
                                if (ch < 7) nxt = *reinterpret_cast<const uint4*>(sV + a * 8192 + swz(j, ch + 1));
                                float v8[8];
                                unpack4_bf16(make_uint2(raw.x, raw.y), *reinterpret_cast<float(*)[4]>(&v8[0]));
                                unpack4_bf16(make_uint2(raw.z, raw.w), *reinterpret_cast<float(*)[4]>(&v8[4]));
#pragma unroll
                                for (int i = 0; i < 8; ++i) v8[i] -= z[8 * ch + i];
                                *reinterpret_cast<uint4*>(sV + a * 8192 + swz(j, ch)) = pack8(v8);
                            }
                        }
                    }
                    KDA_TC_PHASE(19);
                }
            }
            sync_compute();
            KDA_TC_PHASE(9);
            // 16 -> 32: blocks (1,0) and (3,2).  thread: block b, row r, columns m2, m2+1
            {
                const int b = tid >> 7, r = (tid >> 3) & 15, m2 = (tid & 7) * 2;
                const int o0 = 32 * b, o1 = o0 + 16;
                float arow[16];
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(&arow[j]) = *reinterpret_cast<const float4*>(&Am[(o1 + r) * AS + o0 + j]);
                float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    const float2 t2 = *reinterpret_cast<const float2*>(&Tm[(o0 + j) * AS + o0 + m2]);
                    const float2 t3 = *reinterpret_cast<const float2*>(&Tm[(o0 + j + 1) * AS + o0 + m2]);
                    x0 = fmaf(arow[j], t2.x, x0); x1 = fmaf(arow[j], t2.y, x1);
                    x2 = fmaf(arow[j + 1], t3.x, x2); x3 = fmaf(arow[j + 1], t3.y, x3);
                }
                x0 += x2; x1 += x3;
                *reinterpret_cast<float2*>(&Xs[(16 * b + r) * 36 + m2]) = make_float2(x0, x1);
                sync_compute();
                float y0 = 0.f, y1 = 0.f;
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const float tz = Tm[(o1 + r) * AS + o1 + jj];
                    const float2 xx = *reinterpret_cast<const float2*>(&Xs[(16 * b + jj) * 36 + m2]);
                    y0 = fmaf(tz, xx.x, y0); y1 = fmaf(tz, xx.y, y1);
                }
                *reinterpret_cast<float2*>(&Tm[(o1 + r) * AS + o0 + m2]) = make_float2(-y0, -y1);
            }
            sync_compute();
            KDA_TC_PHASE(10);
            // 32 -> 64 on the tensor cores (tf32): X^T = T0^T A10^T, then Y^T = X^T T1^T with
            // X^T read back from TMEM by the second MMA; Tinv[32:64, 0:32] = -Y.  Operands:
            // fp32 K-major tiles written here (T1 serves as the second product's B).
            {
                uint8_t* t0t = sX + X_T0T;
                uint8_t* t1 = sX + X_T1;
                const int rw = tid >> 3, k4 = (tid & 7) * 4;       // row 0..31, 4 columns
                float4 c4;
                c4.x = Tm[(k4 + 0) * AS + rw]; c4.y = Tm[(k4 + 1) * AS + rw];
                c4.z = Tm[(k4 + 2) * AS + rw]; c4.w = Tm[(k4 + 3) * AS + rw];
                *reinterpret_cast<float4*>(t0t + f32_off(rw, k4)) = c4;                 // T0^T[m][j]
                *reinterpret_cast<float4*>(t1 + f32_off(rw, k4)) =
                    *reinterpret_cast<const float4*>(&Tm[(32 + rw) * AS + 32 + k4]);  // T1[r][jj]
                *reinterpret_cast<float4*>(sX + X_A10 + f32_off(rw, k4)) =
                    *reinterpret_cast<const float4*>(&Am[(32 + rw) * AS + k4]);       // A10[r][j]
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            wait_mma();
            // both products are done: Y^T = X^T T1^T is in TMEM (M=64 rows c = 16 q4 + lane,
            // columns r'); Tinv[32 + r', c] = -Y[r', c]
            if (q4 < 2) {
                float v[32];
                tmem_ld16(tmem + tlane + TM_WK + 32, *reinterpret_cast<float(*)[16]>(&v[0]));
                tmem_ld16(tmem + tlane + TM_WK + 48, *reinterpret_cast<float(*)[16]>(&v[16]));
                tmem_wait_ld();
                if (hf == 0 && lane < 16) {
                    const int c = 16 * q4 + lane;
#pragma unroll
                    for (int r = 0; r < 32; ++r) Tm[(32 + r) * AS + c] = -v[r];
                }
            }
            tc_fence_before();
            sync_compute();
            KDA_TC_PHASE(11);
            // Tb = Tinv diag(beta) as the K-major A operand [64 r][64 m]; zero above the diagonal
            uint8_t* sTB = sX + X_TB;
#pragma unroll
            for (int rep = 0; rep < 2; ++rep) {
                const int e = tid + NT * rep;
                const int jr = e & 63, ch = e >> 6;
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int m = 8 * ch + i;
                    v[i] = (jr >= m) ? Tm[jr * AS + m] * sBeta[m] : 0.0f;
                }
                *reinterpret_cast<uint4*>(sTB + swz(jr, ch)) = pack8(v);
                if constexpr (kRecord) {   // T itself, in the same K-major layout
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int m = 8 * ch + i;
                        v[i] = (jr >= m) ? Tm[jr * AS + m] : 0.0f;
                    }
                    *reinterpret_cast<uint4*>(rec_of(chunk) + bwdrec::T + swz(jr, ch)) = pack8(v);
                }
            }
            KDA_TC_PHASE(12);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        KDA_TC_PHASE(4);
        if constexpr (kSummary) {
        // ================= W = Tb (k*gamma)   (M=64, N=128, K=64)
        wait_mma();
        {
            // -W as the K-major A operand of the U MMA; M=64 rows m = 16 q4 + lane (lane < 16)
            float v[64];
            tmem_ld64(tmem + tlane + TM_WK + 64 * hf, v);
            if (lane < 16) {
                const int m = 16 * q4 + lane;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float w8[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) w8[i] = -v[8 * ch + i];
                    *reinterpret_cast<uint4*>(sX + X_WQ + hf * 8192 + swz(m, ch)) = pack8(w8);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        }

        KDA_TC_PHASE(5);
        if constexpr (kSummary) {
        // ================= [U_M | U_N] = -W [M | N] + [0 | Tb V]   (M=64, N=256, K=128 (+64))
        // (the decay of [M | N] was applied beside the [A/beta ; P] product)
        wait_mma();
        if (tid < C) {
            const int64_t nxt = (int64_t)(chunk + 1) * C + tid;   // token index in the segment
            beta_next = nxt < len ? load_beta(nxt) : 0.0f;
        }
        {   // U rows j = 16 q4 + lane: MN-major B [64 j][256 n], four 8 KB atoms
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float v[64];
                tmem_ld64(tmem + tlane + TM_WK + 128 * hf + 64 * p, v);
                if (lane < 16) {
                    const int j = 16 * q4 + lane;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        *reinterpret_cast<uint4*>(sX + X_U + (2 * hf + p) * 8192 + swz(j, ch)) =
                            pack8(&v[8 * ch]);
                }
            }
        }
        KDA_TC_PHASE(6);
        // (the control warp then issues [M | N] += (k*eta)^T [U_M | U_N])
        } else {
        // ================= U = Tb (V - (k*gamma) S)   (issued by the control warp; the decay
        // of S was applied beside the [A/beta ; P] product)
        wait_mma();
        if (tid < C) {
            const int64_t nxt = (int64_t)(chunk + 1) * C + tid;   // token index in the segment
            beta_next = nxt < len ? load_beta(nxt) : 0.0f;
        }
        {   // U as the MN-major B operand [64 j][128 n]: rows j = 16 q4 + lane (lane < 16)
            float v[64];
            tmem_ld64(tmem + tlane + TM_U + 64 * hf, v);
            if (lane < 16) {
                const int j = 16 * q4 + lane;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4*>(sX + X_U + hf * 8192 + swz(j, ch)) = pack8(&v[8 * ch]);
            }
        }
        KDA_TC_PHASE(6);
        // (the control warp then issues S += (k*eta)^T U and O += P U)
        }
        // U is handed over; every thread leaves together on a timeout
        fence_async_smem();
        tc_fence_before();
        const int any_timeout = __syncthreads_or(!ok);
        tc_fence_after();
        KDA_TC_PHASE(8);
        if (any_timeout) {
            broke = true;
            break;
        }
    }

    // ---- the control warp: one thread issues every copy and MMA group at the barriers
    // where the compute warps hand over their operands, and waits for each committed
    // group in order.  Groups without a commit ride on the next group's commit (the
    // tensor pipe runs one thread's MMAs in issue order).
    //   barrier A (operands of [A/beta ; P]):  [A/beta ; P] (commit); forward: (k*gamma) S_start
    //                                            (own barrier), then (q*gamma) S_start; dual:
    //                                            the previous chunk's [Qg | O0] stores, then the
    //                                            loads of this chunk's v and the next q there
    //   barrier B (tf32 solve operands):          the two chained 32 -> 64 solve products
    //                                            (the second reads the first from TMEM; commit)
    //   barrier D (Tb):                          forward: U = Tb (V - (k*gamma) S) (commit);
    //                                            summary: W = Tb (k*gamma) (commit), then Tb V
    //                                            (dual: its own commit, then the next alpha load)
    //   barrier E (-W, summary only):            [U_M | U_N] += -W [M | N] (commit)
    //   barrier F (U):                           S += (k*eta)^T U and O += P U (commit); dual:
    //                                            [M | N] += (k*eta)^T [U_M | U_N] and
    //                                            [Qg | O0] = (q*gamma) [M | N] + P [U_M | U_N]
    const uint32_t idM64 = idesc_bf16(64, 128, false, true);   // M=64, N=128, B MN-major
    auto mma_ap = [&]() {
        const uint32_t l0 = smem_u32(sX + X_L), r0 = smem_u32(sX + X_R);
        constexpr uint32_t idesc = idesc_bf16(128, 96);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_WK, sdesc_sw128(l0 + (ks >> 2) * 16384u + (ks & 3) * 32u),
                     sdesc_sw128(r0 + (ks >> 2) * 12288u + (ks & 3) * 32u), idesc, ks > 0);
        if constexpr (!kRecord) commit_mma();   // record mode commits after its copies
    };
    auto mma_z = [&]() {   // (k*gamma) S_start into U's columns (own barrier)
        const uint32_t kg = smem_u32(sKT), s0 = smem_u32(sS);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_U, sdesc_sw128(kg + (ks >> 2) * 8192 + (ks & 3) * 32),
                     sdesc_sw128(s0 + ks * 2048, 1024, 16384), idM64, ks > 0);
        commit_z();
    };
    auto mma_qs = [&](uint8_t* sQc) {   // O = (q*gamma) S_start (no commit)
        const uint32_t qg = smem_u32(sQc), s0 = smem_u32(sS);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_O, sdesc_sw128(qg + (ks >> 2) * 8192 + (ks & 3) * 32),
                     sdesc_sw128(s0 + ks * 2048, 1024, 16384), idM64, ks > 0);
    };
    auto mma_tf1 = [&]() {   // X^T = T0^T A10^T (no commit: the second product's covers it)
        constexpr uint32_t idesc = idesc_tf32(64, 32);
        const uint32_t a0 = smem_u32(sX + X_T0T), b0 = smem_u32(sX + X_A10);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_tf32(tmem + TM_WK, sdesc_sw128(a0 + ks * 32), sdesc_sw128(b0 + ks * 32), idesc, ks > 0);
    };
    auto mma_tf2 = [&]() {   // Y^T = X^T T1^T with X^T taken from TMEM (the first product)
        constexpr uint32_t idesc = idesc_tf32(64, 32);
        const uint32_t b0 = smem_u32(sX + X_T1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_tf32_ts(tmem + TM_WK + 32, tmem + TM_WK + 8 * ks, sdesc_sw128(b0 + ks * 32), idesc,
                        ks > 0);
        commit_mma();
    };
    auto mma_w = [&]() {
        const uint32_t a0 = smem_u32(sX + X_TB), b0 = smem_u32(sKT);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(tmem + TM_WK, sdesc_sw128(a0 + ks * 32), sdesc_sw128(b0 + ks * 2048, 1024, 8192),
                     idM64, ks > 0);
        commit_mma();
    };
    auto mma_tbv = [&]() {   // Tb V into U (or U_N) (no commit)
        const uint32_t tb = smem_u32(sX + X_TB), v0 = smem_u32(sV);
        const uint32_t d = tmem + (kSummary ? TM_WK + 128 : TM_U);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(d, sdesc_sw128(tb + ks * 32), sdesc_sw128(v0 + ks * 2048, 1024, 8192), idM64, ks > 0);
    };
    auto mma_u = [&]() {   // summary: U_M = -W M (fresh, over W's accumulator), U_N += -W N
        const uint32_t wq = smem_u32(sX + X_WQ), s0 = smem_u32(sS);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_WK, sdesc_sw128(wq + (ks >> 2) * 8192 + (ks & 3) * 32),
                     sdesc_sw128(s0 + ks * 2048, 1024, 16384), idM64, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_WK + 128, sdesc_sw128(wq + (ks >> 2) * 8192 + (ks & 3) * 32),
                     sdesc_sw128(s0 + 32768 + ks * 2048, 1024, 16384), idM64, 1);
        commit_mma();
    };
    auto mma_s = [&](uint8_t* sQc) {
        const uint32_t kh = smem_u32(sKH), u0 = smem_u32(sX + X_U);
        if constexpr (kSummary) {
            constexpr uint32_t idesc = idesc_bf16(128, 256, true, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_S, sdesc_sw128(kh + ks * 2048, 1024, 8192),
                         sdesc_sw128(u0 + ks * 2048, 1024, 8192), idesc, 1);
            if constexpr (kDual) {
                // [Qg | O0] = (q*gamma) [M | N] + P [U_M | U_N]   (M=64, N=256) over the scratch
                // and U columns, which the [U_M | U_N] extraction has emptied; [M | N] is read
                // from its bf16 copy, still the chunk's start value
                constexpr uint32_t id_o = idesc_bf16(64, 256, false, true);
                const uint32_t qg = smem_u32(sQc), s0 = smem_u32(sS), p0 = smem_u32(sX + X_P);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tmem + TM_WK, sdesc_sw128(qg + (ks >> 2) * 8192 + (ks & 3) * 32),
                             sdesc_sw128(s0 + ks * 2048, 1024, 16384), id_o, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_WK, sdesc_sw128(p0 + ks * 32),
                             sdesc_sw128(u0 + ks * 2048, 1024, 8192), id_o, 1);
            }
        } else {
            constexpr uint32_t id_s = idesc_bf16(128, 128, true, true);
            const uint32_t p0 = smem_u32(sX + X_P);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_S, sdesc_sw128(kh + ks * 2048, 1024, 8192),
                         sdesc_sw128(u0 + ks * 2048, 1024, 8192), id_s, 1);
            if constexpr (!kRecord) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_O, sdesc_sw128(p0 + ks * 32),
                             sdesc_sw128(u0 + ks * 2048, 1024, 8192), idM64, 1);
            }
        }
        if constexpr (!kRecord) commit_mma();   // record mode commits after its copies
    };
    auto handoff = [&]() {
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };
    if (!compute)
    for (int chunk = 0; chunk < nchunks; ++chunk) {
        const int64_t row0 = bos + (int64_t)chunk * C;
        uint8_t* sQc = sQ + (chunk & 1) * 16384;
        if (ctl && chunk > 0) wait_mma();   // the previous chunk's state update (and O)
        handoff();   // A
        if (ctl) {
            KDA_TC_PHASE(20);
            if (ok) {
                if constexpr (kRecord) {   // the tiles the extraction overwrites go first
                    uint8_t* rp = rec_of(chunk);
                    if (h == 0) {
                        const int64_t rem = len - (int64_t)chunk * C;
                        seg.hdr[s_cbase + chunk] = bwdrec::Header{row0, (int32_t)(rem < C ? rem : C), 0};
                    }
                    bulk_store(rp + bwdrec::L, sX + X_L, 32768);
                    bulk_store(rp + bwdrec::R, sX + X_R, 24576);
                    bulk_commit_group();
                }
                mma_ap();
                if (!kSummary) {
                    mma_z();
                    if (!kRecord) mma_qs(sQc);
                }
                if constexpr (kRecord) {   // the tiles are read before anyone may overwrite them
                    bulk_wait_read_all();
                    commit_mma();
                }
            }
            if (!kSummary && !kRecord && chunk > 0) store_o(sQ + ((chunk + 1) & 1) * 16384, row0 - C);
            if (chunk + 1 < nchunks && ok) {   // k and alpha are consumed
                issue_ka(row0 + C);
                issued(tka);
            }
            if (kDual && ok) {
                // the previous chunk (full: only a segment's last chunk is not) leaves from
                // its staging buffers; v and the next q go there once the stores have read them
                if (chunk > 0) {
                    store_dual(sQ + ((chunk + 1) & 1) * 16384, row0 - C);
                    bulk_wait_read_all();
                }
                issue_v(row0);
                issued(tv);
                if (chunk + 1 < nchunks) {
                    issue_q(row0 + C, (chunk + 1) & 1);
                    issued(tq);
                }
            }
            wait_mma();
            KDA_TC_PHASE(21);
            if (!kSummary) {
                // the O store has read its staging buffer: load the next q there
                bulk_wait_read_all();
                if (chunk + 1 < nchunks && ok) {
                    issue_q(row0 + C, (chunk + 1) & 1);
                    issued(tq);
                }
                wait_z();
                KDA_TC_PHASE(22);
            }
        }
        handoff();   // B
        if (ctl) {
            if (kRecord && ok) {   // tiles that stay valid until the next chunk's gate phase
                uint8_t* rp = rec_of(chunk);   // (their reads are waited for before later commits)
                bulk_store(rp + bwdrec::P, sX + X_P, 8192);
                bulk_store(rp + bwdrec::S, sS, 32768);
                bulk_store(rp + bwdrec::QT, sQc, 16384);
                bulk_store(rp + bwdrec::KT, sKT, 16384);
                bulk_store(rp + bwdrec::KH, sKH, 16384);
                bulk_commit_group();
            }
            if (ok) {
                mma_tf1();
                mma_tf2();
            }
            wait_mma();
        }
        handoff();   // D
        if (ctl) {
            KDA_TC_PHASE(23);
            if constexpr (kSummary) {
                if (ok) mma_w();
                wait_load(barV, tv);
                if (ok) mma_tbv();
                if (kDual && ok) commit_z();   // Tb V done: alpha may take the buffer
            } else if (ok) {
                if constexpr (kRecord) {
                    bulk_store(rec_of(chunk) + bwdrec::RV, sV, 16384);
                    bulk_commit_group();
                }
                mma_tbv();   // U = Tb (V - (k*gamma) S), the v tile holding the difference
                if constexpr (kRecord) bulk_wait_read_all();   // before the next v load
                commit_mma();
            }
            wait_mma();
            if constexpr (kDual) {
                wait_z();
                if (chunk + 1 < nchunks && ok) {
                    issue_al(row0 + C);
                    issued(tal);
                }
            }
            KDA_TC_PHASE(24);
        }
        if constexpr (kSummary) {
            handoff();   // E
            if (ctl) {
                if (ok) mma_u();
                wait_mma();
            }
        }
        if (!kDual && ctl && chunk + 1 < nchunks && ok) {   // v is consumed
            issue_v(row0 + C);
            issued(tv);
        }
        tc_fence_before();
        const int any_timeout = __syncthreads_or(!ok);   // F, uniform: every thread leaves together
        tc_fence_after();
        if (any_timeout) {
            broke = true;
            break;
        }
        if (ctl && ok) {
            if constexpr (kRecord) {
                bulk_store(rec_of(chunk) + bwdrec::U, sX + X_U, 16384);
                bulk_commit_group();
            }
            mma_s(sQc);
            if constexpr (kRecord) {
                bulk_wait_read_all();
                commit_mma();
            }
        }
    }
    if (ctl && nchunks > 0 && !broke) wait_mma();

    // the last chunk's state update and outputs (staged in the q buffer it did not use)
    const int last_Lc = nchunks > 0 ? (int)(len - (int64_t)(nchunks - 1) * C) : 0;
    uint8_t* last_stage = sQ + (nchunks & 1) * 16384;
    if (compute && nchunks > 0 && !broke)
        finish_prev(bos + (int64_t)(nchunks - 1) * C, last_Lc, last_stage);
    fence_async_smem();

    if (!ok) atomicExch(sFlag, 1);
    __syncthreads();
    if ((!kSummary || kDual) && ctl) {
        if (!kRecord && nchunks > 0 && !broke && !*sFlag && last_Lc == C) {
            if constexpr (kDual) store_dual(last_stage, bos + (int64_t)(nchunks - 1) * C);
            else store_o(last_stage, bos + (int64_t)(nchunks - 1) * C);
        }
        bulk_wait_all();   // every O store has completed before shared memory is released
    }
    if (*sFlag && ctl) {
        // a wait gave up: let this CTA's own copies and MMAs in flight finish (bounded)
        // before its shared and tensor memory are released.  The control thread issues
        // every copy and MMA group and waits for each group in order; a load stream's
        // last copy completes the phase of parity (issued - 1) & 1.
        if (tq.issued) mbar_wait_ns(barQ, (tq.issued - 1) & 1u, kWaitNs);
        if (tka.issued) mbar_wait_ns(barKA, (tka.issued - 1) & 1u, kWaitNs);
        if (tv.issued) mbar_wait_ns(barV, (tv.issued - 1) & 1u, kWaitNs);
        if (tal.issued) mbar_wait_ns(barAl, (tal.issued - 1) & 1u, kWaitNs);
        if (mma_out) mbar_wait_ns(barM, mma_out_ph, kWaitNs);
        if (z_out) mbar_wait_ns(barZ, z_out_ph, kWaitNs);
    }
    __syncthreads();
    if (kCtaStatus && tid == 0) status[(size_t)n * H + h] = *sFlag;
    if (*sFlag) {
        if (!kCtaStatus && tid == 0) atomicExch(status, 1);
    } else if (!compute) {
    } else if (kSummary) {
        const int c = 32 * q4 + lane;
        float* dst = seg.maps + ((((size_t)n * seg.per_seq + gseg) * H + h) * DK + c) * (DK + DV) +
                     128 * hf;
#pragma unroll
        for (int blk = 0; blk < 8; ++blk) {
            float v[16];
            tmem_ld16(tmem + tlane + TM_S + 128 * hf + 16 * blk, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(dst + 16 * blk + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    } else if (S_final && last_seg && slot_ok) {
        const int c = 32 * q4 + lane;
        float* dst = S_final + (((size_t)slot * H + h) * DK + c) * DV + 64 * hf;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            float v[16];
            tmem_ld16(tmem + tlane + TM_S + 64 * hf + 16 * blk, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(dst + 16 * blk + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// S_{g+1} = M_g S_g + N_g over the segments of one sequence, in fp32: one CTA
// per (16 value columns, head, sequence), thread i owns row i of the state.
// start[g = 0] receives S0 (or zeros), so no later kernel reads S0 and S_final
// may alias S0.  maps holds nmaps maps per sequence: nseg - 1 (the last segment's
// is not needed), or nseg, and then S_final (if not null) receives the state after
// the last segment.
constexpr int SCAN_COLS = 16;
__global__ void __launch_bounds__(DK)
kda_segment_scan_kernel(const float* S0, const float* __restrict__ maps, float* __restrict__ start,
                        int nseg, int nmaps, int H, float* S_final) {
    __shared__ __align__(16) float sS[DK][SCAN_COLS];
    const int cb = blockIdx.x, h = blockIdx.y, n = blockIdx.z, i = threadIdx.x;
    const size_t col = (size_t)SCAN_COLS * cb;
    float cur[SCAN_COLS];
    const float* src = S0 ? S0 + (((size_t)n * H + h) * DK + i) * DV + col : nullptr;
#pragma unroll
    for (int c = 0; c < SCAN_COLS; c += 4) {
        const float4 f = src ? *reinterpret_cast<const float4*>(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        cur[c] = f.x; cur[c + 1] = f.y; cur[c + 2] = f.z; cur[c + 3] = f.w;
    }
    for (int g = 0; g < nseg; ++g) {
        float* dst = start + ((((size_t)n * nseg + g) * H + h) * DK + i) * DV + col;
#pragma unroll
        for (int c = 0; c < SCAN_COLS; c += 4)
            *reinterpret_cast<float4*>(dst + c) = make_float4(cur[c], cur[c + 1], cur[c + 2], cur[c + 3]);
        if (g == nmaps) break;
        __syncthreads();   // the previous step's reads of sS are done
#pragma unroll
        for (int c = 0; c < SCAN_COLS; ++c) sS[i][c] = cur[c];
        __syncthreads();
        const float* Mrow = maps + ((((size_t)n * nmaps + g) * H + h) * DK + i) * (DK + DV);
#pragma unroll
        for (int c = 0; c < SCAN_COLS; ++c) cur[c] = Mrow[DK + col + c];   // N_g
        for (int j = 0; j < DK; j += 4) {
            const float4 m = *reinterpret_cast<const float4*>(Mrow + j);
            const float mj[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
                for (int c = 0; c < SCAN_COLS; c += 4) {
                    const float4 sv = *reinterpret_cast<const float4*>(&sS[j + jj][c]);
                    cur[c] = fmaf(mj[jj], sv.x, cur[c]);
                    cur[c + 1] = fmaf(mj[jj], sv.y, cur[c + 1]);
                    cur[c + 2] = fmaf(mj[jj], sv.z, cur[c + 2]);
                    cur[c + 3] = fmaf(mj[jj], sv.w, cur[c + 3]);
                }
            }
        }
    }
    if (nmaps == nseg && S_final) {
        float* dst = S_final + (((size_t)n * H + h) * DK + i) * DV + col;
#pragma unroll
        for (int c = 0; c < SCAN_COLS; c += 4)
            *reinterpret_cast<float4*>(dst + c) = make_float4(cur[c], cur[c + 1], cur[c + 2], cur[c + 3]);
    }
}

// out = the state after maps 0..G-1 applied in order to S0 (S <- M_g S + N_g), fp32.
// maps: [G][nseq][H][DK][DK + DV] (one map per segment, e.g. one per rank); S0 and out:
// [nseq][H][DK][DV] (S0 may be null = 0, out may alias S0: each CTA reads its own
// 16 columns before it writes them).
__global__ void __launch_bounds__(DK)
kda_apply_maps_kernel(const float* S0, const float* __restrict__ maps, int G, int nseq, int H,
                      float* out) {
    __shared__ __align__(16) float sS[DK][SCAN_COLS];
    const int cb = blockIdx.x, h = blockIdx.y, n = blockIdx.z, i = threadIdx.x;
    const size_t col = (size_t)SCAN_COLS * cb;
    float cur[SCAN_COLS];
    const float* src = S0 ? S0 + (((size_t)n * H + h) * DK + i) * DV + col : nullptr;
#pragma unroll
    for (int c = 0; c < SCAN_COLS; c += 4) {
        const float4 f = src ? *reinterpret_cast<const float4*>(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        cur[c] = f.x; cur[c + 1] = f.y; cur[c + 2] = f.z; cur[c + 3] = f.w;
    }
    for (int g = 0; g < G; ++g) {
        __syncthreads();   // the previous step's reads of sS are done
#pragma unroll
        for (int c = 0; c < SCAN_COLS; ++c) sS[i][c] = cur[c];
        __syncthreads();
        const float* Mrow = maps + ((((size_t)g * nseq + n) * H + h) * DK + i) * (DK + DV);
#pragma unroll
        for (int c = 0; c < SCAN_COLS; ++c) cur[c] = Mrow[DK + col + c];   // N_g
        for (int j = 0; j < DK; j += 4) {
            const float4 m = *reinterpret_cast<const float4*>(Mrow + j);
            const float mj[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
                for (int c = 0; c < SCAN_COLS; c += 4) {
                    const float4 sv = *reinterpret_cast<const float4*>(&sS[j + jj][c]);
                    cur[c] = fmaf(mj[jj], sv.x, cur[c]);
                    cur[c + 1] = fmaf(mj[jj], sv.y, cur[c + 1]);
                    cur[c + 2] = fmaf(mj[jj], sv.z, cur[c + 2]);
                    cur[c + 3] = fmaf(mj[jj], sv.w, cur[c + 3]);
                }
            }
        }
    }
    float* dst = out + (((size_t)n * H + h) * DK + i) * DV + col;
#pragma unroll
    for (int c = 0; c < SCAN_COLS; c += 4)
        *reinterpret_cast<float4*>(dst + c) = make_float4(cur[c], cur[c + 1], cur[c + 2], cur[c + 3]);
}

// o += Qg S_g over the tokens of segment g: the last step of the split forward, whose
// dual-mode pass left each segment's zero-start output O0 in o and its map rows Qg.
// One CTA per (slice of up to CR_TILES 128-token tiles of a segment, head, sequence *
// nseg + g), 128 threads, thread 0 issuing every copy and product.  S_g (fp32, from
// the scan) becomes a bf16 MN-major B operand once; each tile of Qg (K-major A) gives
// one M=128, N=128, K=128 product in TMEM (two accumulators, so that the next tile's
// product runs beside this tile's additions); thread t adds row t of it to row t of
// the o tile in shared memory, and the tile leaves by TMA store.  Qg and o tiles
// arrive by TMA in three stages each, issued two to three tiles ahead: the pass is
// bound by memory (256 bytes read twice and written once per token and head).  A
// segment's ragged last tile is written row by row (a TMA box would spill into the
// next segment's rows, which another CTA writes).
constexpr int CR_TILE = 128;
constexpr int CR_TILES = 64;
constexpr int CR_THREADS = 128;
constexpr int CR_STAGES = 3;
constexpr uint32_t CR_OFF_S = 0;          // S_g bf16 [128 c][128 n], two [128][64] atoms
constexpr uint32_t CR_OFF_G = 32768;      // Qg tiles [128 t][128 c] (two [128][64] atoms), 3 stages
constexpr uint32_t CR_OFF_O = CR_OFF_G + CR_STAGES * 32768;   // o tiles, same layout, 3 stages
constexpr uint32_t CR_OFF_BAR = CR_OFF_O + CR_STAGES * 32768; // uint64 x8: Qg (3), o (3), MMA (2)
constexpr uint32_t CR_OFF_TMEM = CR_OFF_BAR + 64;
constexpr uint32_t CR_SMEM = CR_OFF_TMEM + 16 + 1024;
static_assert(CR_SMEM <= 232448, "correction kernel shared memory");

__global__ void __launch_bounds__(CR_THREADS, 1)
kda_segment_correct_kernel(const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmO,
                           const float* __restrict__ start, const int32_t* __restrict__ cu_seqlens,
                           int64_t T, int H, int nseg, int skip_first, __nv_bfloat16* __restrict__ out,
                           int* status) {
    const int h = blockIdx.y, z = blockIdx.z, n = z / nseg, g = z % nseg;
    if (skip_first && g == 0) return;   // S_0 = 0: nothing to add
    int64_t bos, len;
    seq_range(cu_seqlens, n, T, bos, len);
    const int64_t nch = (len + C - 1) / C, cps = (nch + nseg - 1) / nseg;
    const int64_t t1 = min(min((int64_t)(g + 1) * cps, nch) * C, len);
    const int64_t s0 = min(min((int64_t)g * cps, nch) * C, len) + (int64_t)blockIdx.x * CR_TILES * CR_TILE;
    if (s0 >= t1) return;   // (uniform over the CTA)
    const int ntiles = (int)min((int64_t)CR_TILES, (t1 - s0 + CR_TILE - 1) / CR_TILE);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* barG = reinterpret_cast<uint64_t*>(sm + CR_OFF_BAR);
    uint64_t* barO = barG + 3;
    uint64_t* barM = barG + 6;
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + CR_OFF_TMEM);
    __shared__ int s_fail;
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        for (int i = 0; i < 8; ++i) mbar_init(barG + i, 1);
        mbar_fence_init();
        s_fail = 0;
    }
    if (warp == 0) tmem_alloc(sTmem, 256);
    auto tile_row = [&](int i) { return (int)(bos + s0 + (int64_t)i * CR_TILE); };
    auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int i) {
        mbar_arrive_expect_tx(bar, 32768);
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 2; ++b)
                tma_load_2d(dst + a * 16384 + b * 8192, map, bar, h * DK + 64 * a, tile_row(i) + 64 * b);
    };
    auto issue_g = [&](int i) { load_tile(&tmG, sm + CR_OFF_G + (i % 3) * 32768, barG + i % 3, i); };
    auto issue_o = [&](int i) { load_tile(&tmO, sm + CR_OFF_O + (i % 3) * 32768, barO + i % 3, i); };
    uint32_t ng[3] = {0, 0, 0}, no[3] = {0, 0, 0};   // (thread 0) loads issued per stage
    __syncthreads();
    if (tid == 0) {
        for (int i = 0; i < ntiles && i < 3; ++i) {
            issue_g(i);
            ++ng[i];
            issue_o(i);
            ++no[i];
        }
    }
    // S_g as bf16: thread c writes row c (both 64-column atoms)
    {
        const float* src = start + (((size_t)z * H + h) * DK + tid) * DV;
#pragma unroll
        for (int blk = 0; blk < DV / 8; ++blk) {
            const float4 f0 = *reinterpret_cast<const float4*>(src + 8 * blk);
            const float4 f1 = *reinterpret_cast<const float4*>(src + 8 * blk + 4);
            const float v[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
            *reinterpret_cast<uint4*>(sm + CR_OFF_S + (blk >> 3) * 16384 + swz(tid, blk & 7)) = pack8(v);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t tl = (uint32_t)(32 * warp) << 16;
    bool ok = true;
    bool mma_out = false;   // (thread 0) a product committed and not yet seen complete
    uint32_t mma_ph = 0, mma_b = 0;
    auto product = [&](int i) {   // thread 0: tile i's product into accumulator i & 1
        if (ok && !mbar_wait_ns(barG + i % 3, (uint32_t)(i / 3) & 1u, kWaitNs)) ok = false;
        tc_fence_after();
        if (!ok) return;
        constexpr uint32_t id = idesc_bf16(128, 128, false, true);
        const uint32_t a0 = smem_u32(sm + CR_OFF_G + (i % 3) * 32768), b0 = smem_u32(sm + CR_OFF_S);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + 128 * (i & 1), sdesc_sw128(a0 + (ks >> 2) * 16384 + (ks & 3) * 32),
                     sdesc_sw128(b0 + ks * 2048, 1024, 16384), id, ks > 0);
        mma_commit(barM + (i & 1));
        mma_out = true;
        mma_ph = (uint32_t)(i >> 1) & 1u;
        mma_b = (uint32_t)(i & 1);
    };
    if (tid == 0 && ntiles > 0) product(0);
    for (int i = 0; i < ntiles; ++i) {
        // tile i's product is done: its Qg stage is free, the next product may start
        bool w = __syncthreads_and(ok) && mbar_wait_ns(barM + (i & 1), (uint32_t)(i >> 1) & 1u, kWaitNs);
        tc_fence_after();
        if (!__syncthreads_and(w)) { ok = false; break; }
        if (tid == 0) {
            mma_out = false;
            if (i + 3 < ntiles) { issue_g(i + 3); ++ng[i % 3]; }
            if (i + 1 < ntiles) product(i + 1);
        }
        // row tid of the product onto row tid of the o tile
        w = mbar_wait_ns(barO + i % 3, (uint32_t)(i / 3) & 1u, kWaitNs);
        if (!__syncthreads_and(w)) { ok = false; break; }
        const int64_t t = s0 + (int64_t)i * CR_TILE + tid;
        const bool full = s0 + (int64_t)(i + 1) * CR_TILE <= t1;
        uint8_t* ot = sm + CR_OFF_O + (i % 3) * 32768;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            float acc[32];
            tmem_ld32(tmem + tl + 128 * (i & 1) + 32 * p, acc);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint8_t* cell = ot + (p >> 1) * 16384 + swz(tid, 4 * (p & 1) + ch);
                const uint4 raw = *reinterpret_cast<const uint4*>(cell);
                const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
                float v[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wds[e]));
                    v[2 * e] = f.x + acc[8 * ch + 2 * e];
                    v[2 * e + 1] = f.y + acc[8 * ch + 2 * e + 1];
                }
                const uint4 res = pack8(v);
                if (full) {
                    *reinterpret_cast<uint4*>(cell) = res;
                } else if (t < t1) {
                    reinterpret_cast<uint4*>(out + ((size_t)(bos + t) * H + h) * DV)[8 * (p >> 1) + 4 * (p & 1) + ch] = res;
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            if (full) {
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int b = 0; b < 2; ++b)
                        tma_store_2d(&tmO, ot + a * 16384 + b * 8192, h * DV + 64 * a, tile_row(i) + 64 * b);
                bulk_commit_group();
            }
            // the o stage of tile i - 1 has been read by its store: tile i + 2 goes there
            if (i >= 1 && i + 2 < ntiles) {
                if (full) bulk_wait_read_1();   // (the store just issued may still be reading)
                else bulk_wait_read_all();
                issue_o(i + 2);
                ++no[(i + 2) % 3];
            }
        }
    }
    if (!ok && tid == 0) {   // let this CTA's own copies and product in flight finish (bounded)
        s_fail = 1;
        for (int st = 0; st < 3; ++st) {
            if (ng[st]) mbar_wait_ns(barG + st, (ng[st] - 1) & 1u, kWaitNs);
            if (no[st]) mbar_wait_ns(barO + st, (no[st] - 1) & 1u, kWaitNs);
        }
        if (mma_out) mbar_wait_ns(barM + mma_b, mma_ph, kWaitNs);
    }
    if (tid == 0) bulk_wait_all();   // every o store has completed before shared memory goes
    tc_fence_before();
    __syncthreads();
    if (s_fail && tid == 0) atomicExch(status, 1);
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [rows, H*128] bf16, box 64 x 64, 128-byte swizzle
static bool make_map(CUtensorMap* m, const void* base, int64_t rows, int H) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)H * 128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)H * 128 * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

bool make_tc_maps(TcMaps* m, const void* q, const void* k, const void* v, const void* alpha,
                  const void* out, int64_t rows, int H) {
    return tc::make_map(&m->q, q, rows, H) && tc::make_map(&m->k, k, rows, H) &&
           tc::make_map(&m->a, alpha, rows, H) && tc::make_map(&m->v, v, rows, H) &&
           tc::make_map(&m->o, out ? out : v, rows, H);
}

template <bool kCtaStatus, bool kSummary, bool kFused = false, bool kRecord = false,
          bool kDual = false>
static cudaError_t launch_tc_t(const TcMaps& m, const void* beta, const float* S0, const int32_t* cu,
                               int nseq, void* out, float* S_final, int64_t T, int H, int* status,
                               const tc::Segments& seg, cudaStream_t stream,
                               const CUtensorMap* tmG = nullptr) {
    constexpr uint32_t smem = kDual ? tc::dual::SMEM_BYTES : tc::SMEM_BYTES;
    auto* kern = tc::kda_chunk_tc_kernel<kCtaStatus, kSummary, kFused, kRecord, kDual>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(1, H, nseq * seg.per_seq);
    kern<<<grid, tc::NTHREADS, smem, stream>>>(m.q, m.k, m.a, m.v, m.o, tmG ? *tmG : m.o,
                                               (const __nv_bfloat16*)beta, S0, cu, (__nv_bfloat16*)out,
                                               S_final, T, H, status, seg);
    return cudaGetLastError();
}

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const void* alpha,
                            const void* beta, const float* S0, const int32_t* cu, int nseq,
                            void* out, float* S_final, int64_t rows, int64_t T, int H, int* status,
                            cudaStream_t stream, const int32_t* slots, int num_slots, int fused) {
    TcMaps m;
    if (!make_tc_maps(&m, q, k, v, alpha, out, rows, H)) return cudaErrorInvalidValue;
    const tc::Segments whole{1, 1, nullptr, nullptr, slots, num_slots};
    return fused ? launch_tc_t<false, false, true>(m, beta, S0, cu, nseq, out, S_final, T, H, status,
                                                   whole, stream)
                 : launch_tc_t<false, false>(m, beta, S0, cu, nseq, out, S_final, T, H, status,
                                             whole, stream);
}

// The backward's first pass: the forward recurrence of whole sequences in record mode
// (no outputs), filling rec (one kda_bwd_record.cuh record per (chunk, head), chunks
// numbered across sequences in order) and hdr (one header per chunk; the caller
// zeroes it first, so that unused entries read as empty).
cudaError_t launch_chunk_tc_record(const void* q, const void* k, const void* v, const void* alpha,
                                   const void* beta, const float* S0, const int32_t* cu, int nseq,
                                   int64_t rows, int64_t T, int H, uint8_t* rec,
                                   bwdrec::Header* hdr, int64_t rec_chunks, int* status,
                                   cudaStream_t stream) {
    TcMaps m;
    if (!make_tc_maps(&m, q, k, v, alpha, nullptr, rows, H)) return cudaErrorInvalidValue;
    tc::Segments whole{1, 1, nullptr, nullptr, nullptr, 0};
    whole.rec = rec;
    whole.hdr = hdr;
    whole.rec_chunks = rec_chunks;
    return launch_tc_t<false, false, false, true>(m, beta, S0, cu, nseq, nullptr, nullptr, T, H,
                                                  status, whole, stream);
}

// Bytes of workspace the split forward uses: every segment's map [M | N] and start
// state (fp32), and the map rows Qg of every token (bf16, like the output).
size_t chunk_tc_segmented_workspace_bytes(int64_t nseq, int64_t rows, int H, int nseg) {
    if (nseg < 2) return 0;
    return sizeof(float) * (size_t)nseq * H * nseg * tc::DK * ((tc::DK + tc::DV) + tc::DV) +
           sizeof(__nv_bfloat16) * (size_t)rows * H * tc::DK;
}

// The forward split along time into nseg segments per sequence: three launches.
// (1) Every segment in the dual mode: its map [M | N], its output from a zero start
// state (into out) and its map rows Qg; (2) the fp32 scan of the start states S_g,
// which also gives S_final; (3) o += Qg S_g on the tensor cores.
cudaError_t launch_chunk_tc_segmented(const void* q, const void* k, const void* v,
                                      const void* alpha, const void* beta, const float* S0,
                                      const int32_t* cu, int nseq, void* out, float* S_final,
                                      int64_t rows, int64_t T, int H, int nseg, void* workspace,
                                      int* status, cudaStream_t stream, int fused) {
    if (nseg < 2 || nseq * (int64_t)nseg > 65535) return cudaErrorInvalidValue;
    TcMaps m;
    if (!make_tc_maps(&m, q, k, v, alpha, out, rows, H)) return cudaErrorInvalidValue;
    float* maps = static_cast<float*>(workspace);
    float* start = maps + (size_t)nseq * H * nseg * tc::DK * (tc::DK + tc::DV);
    __nv_bfloat16* qg = reinterpret_cast<__nv_bfloat16*>(start + (size_t)nseq * H * nseg * tc::DK * tc::DV);
    CUtensorMap tmG;
    if (!tc::make_map(&tmG, qg, rows, H)) return cudaErrorInvalidValue;
    tc::Segments dual{nseg, nseg, nullptr, maps};
    dual.qg = qg;
    cudaError_t e = fused ? launch_tc_t<false, true, true, false, true>(m, beta, nullptr, cu, nseq, out,
                                                                        nullptr, T, H, status, dual, stream,
                                                                        &tmG)
                          : launch_tc_t<false, true, false, false, true>(m, beta, nullptr, cu, nseq, out,
                                                                         nullptr, T, H, status, dual, stream,
                                                                         &tmG);
    if (e != cudaSuccess) return e;
    tc::kda_segment_scan_kernel<<<dim3(tc::DV / tc::SCAN_COLS, H, nseq), tc::DK, 0, stream>>>(
        S0, maps, start, nseg, nseg, H, S_final);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc::kda_segment_correct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tc::CR_SMEM);
    if (e != cudaSuccess) return e;
    // slices per segment: a segment holds at most ceil(chunks / nseg) chunks of the longest
    // sequence, which is at most T tokens (packed: the whole batch)
    const int64_t cps = ((T + tc::C - 1) / tc::C + nseg - 1) / nseg;
    const int64_t slice_tokens = (int64_t)tc::CR_TILES * tc::CR_TILE;
    const int64_t nsl = (cps * tc::C + slice_tokens - 1) / slice_tokens;
    const int slices = (int)(nsl > 1 ? nsl : 1);
    tc::kda_segment_correct_kernel<<<dim3(slices, H, nseq * nseg), tc::CR_THREADS, tc::CR_SMEM, stream>>>(
        tmG, m.o, start, cu, T, H, nseg, S0 == nullptr ? 1 : 0, static_cast<__nv_bfloat16*>(out), status);
    return cudaGetLastError();
}

// Segment maps of whole sequences: maps [nseq][H][DK][DK + DV] fp32 with
// S_end = M S_start + N over each sequence's tokens (the summary mode, one segment).
cudaError_t launch_segment_maps(const void* k, const void* v, const void* alpha, const void* beta,
                                const int32_t* cu, int nseq, float* maps, int64_t rows, int64_t T,
                                int H, int* status, cudaStream_t stream) {
    TcMaps m;
    if (!make_tc_maps(&m, k, k, v, alpha, nullptr, rows, H)) return cudaErrorInvalidValue;
    const tc::Segments one{1, 1, nullptr, maps};
    return launch_tc_t<false, true>(m, beta, nullptr, cu, nseq, nullptr, nullptr, T, H, status, one,
                                    stream);
}

cudaError_t launch_apply_maps(const float* S0, const float* maps, int G, int nseq, int H, float* out,
                              cudaStream_t stream) {
    tc::kda_apply_maps_kernel<<<dim3(tc::DV / tc::SCAN_COLS, H, nseq), tc::DK, 0, stream>>>(
        S0, maps, G, nseq, H, out);
    return cudaGetLastError();
}

// Same kernel, one status word per (sequence, head) CTA at status[n * H + h].
cudaError_t launch_chunk_tc_cta_status(const void* q, const void* k, const void* v,
                                       const void* alpha, const void* beta, const float* S0,
                                       const int32_t* cu, int nseq, void* out, float* S_final,
                                       int64_t rows, int64_t T, int H, int* status,
                                       cudaStream_t stream) {
    TcMaps m;
    if (!make_tc_maps(&m, q, k, v, alpha, out, rows, H)) return cudaErrorInvalidValue;
    const tc::Segments whole{1, 1, nullptr, nullptr};
    return launch_tc_t<true, false>(m, beta, S0, cu, nseq, out, S_final, T, H, status, whole,
                                    stream);
}

}  // namespace kda
