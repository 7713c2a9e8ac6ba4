// Per-(chunk, head) record of the tensor-core backward pass (bf16, d_k = d_v = 128,
// C = 64).  The forward kernel in record mode writes the chunk's start state and the
// operand tiles it forms anyway, byte for byte as they sit in its shared memory
// (128-byte swizzled rows, so a raw copy into a 1024-aligned shared buffer is again
// a valid MMA operand); the reverse state-gradient kernel adds the state gradient at
// the chunk's end and dY; the chunk-parallel gradient kernel reads them all.
//
// Tile notation (per chunk, tokens r, j in [0, 64), key channels c, value channels n):
//   lam, rho^0, rho^1, gamma, eta: the forward's decay factors (sub-chunk references
//   15 and 47), T = (I + A)^-1, P the masked intra-chunk scores, U = T diag(beta) R,
//   R = V - (k*gamma) S.
#pragma once

#include <stdint.h>

namespace kda {
namespace bwdrec {

constexpr uint32_t S = 0;          // S at the chunk start, bf16 [128 c][128 n] (two [128][64] atoms)
constexpr uint32_t L = 32768;      // [k*lam ; q*lam] bf16 [128 r][128 c] (two [128][64] atoms)
constexpr uint32_t R = 65536;      // [k*rho^0 ; k*rho^1] bf16 [96][128 c] (two [96][64] atoms)
constexpr uint32_t QT = 90112;     // q*gamma bf16 [64 r][128 c] (two [64][64] atoms)
constexpr uint32_t KT = 106496;    // k*gamma
constexpr uint32_t KH = 122880;    // k*eta
constexpr uint32_t P = 139264;     // P bf16 [64 r][64 j]
constexpr uint32_t T = 147456;     // T = (I + A)^-1 bf16 [64 j][64 m] (lower triangle)
constexpr uint32_t RV = 155648;    // R = V - (k*gamma) S bf16 [64 j][128 n] (two [64][64] atoms)
constexpr uint32_t U = 172032;     // U bf16 [64 j][128 n] (two [64][64] atoms)
constexpr uint32_t GC = 188416;    // gamma_C fp32 [128]
constexpr uint32_t DS = 189440;    // dL/dS at the chunk end, bf16 [128 c][128 n]
constexpr uint32_t DY = 222208;    // dY = T^T dU, bf16 [64 m][128 n] (two [64][64] atoms)
constexpr uint32_t BYTES = 238592; // record size (a multiple of 1024)

// One per chunk (not per head): the chunk's first row in the [rows, H, d] arrays and
// its token count (0: no such chunk).
struct Header {
    int64_t row0;
    int32_t len;
    int32_t pad;
};

}  // namespace bwdrec
}  // namespace kda
