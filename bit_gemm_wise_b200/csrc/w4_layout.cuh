// Kernel layouts of a prepacked INT4 weight (internal; the ABI treats them as opaque).
//
// Both layouts hold exactly the canonical codes, fp16 scales and int16 zeros, only moved:
// "Four-bit inference ... Tahoma", MSE clipping -- portable codes, scales and zero terms are
// rearranged once into a GPU-specific layout, without dequantizing or requantizing.
#pragma once
#include <stdint.h>
#include <stddef.h>

namespace w4 {

// ---------------------------------------------------------------- W4_LAYOUT_GEMV
// The weight is cut into units of 8 rows x 128 k ("octet x unit"). N is padded to a
// multiple of 8 and K to a multiple of 128 with code 0, scale 0.
//   codes:  [N8 = Npad/8][U = Kpad/128][32 lanes][4 words], 512 bytes per unit. Lane
//           t = 4r + c owns row r of the octet and the 32-wide chunk c of the unit; word w
//           holds k = 128u + 32c + 8w + (0..7) with q[k0 + 2i] in bits [4i, 4i+4) and
//           q[k0 + 2i + 1] in bits [16 + 4i, 20 + 4i), i = 0..3, so that masking the word
//           (shifted by 4i) with 0x000F000F lines up two codes with one bf16x2 pair of x.
//   scales: [N8][U][8 rows][128/g] u32, lo 16 bits the fp16 scale, hi 16 bits the zero
//           (8 for symmetric weights). One octet's scales are contiguous (TMA-staged).
struct GemvLayout {
    int64_t N, K, Npad, Kpad, N8, U;
    int g;
    size_t codes_bytes, scales_bytes, total;
};

inline GemvLayout gemv_layout(int64_t N, int64_t K, int g) {
    GemvLayout L;
    L.N = N; L.K = K; L.g = g;
    L.Npad = (N + 7) / 8 * 8;
    L.Kpad = (K + 127) / 128 * 128;
    L.N8 = L.Npad / 8;
    L.U = L.Kpad / 128;
    L.codes_bytes = (size_t)L.Npad * (size_t)L.Kpad / 2;
    L.scales_bytes = (size_t)L.Npad * (size_t)(L.Kpad / g) * 4;
    L.total = L.codes_bytes + L.scales_bytes;
    return L;
}

// ---------------------------------------------------------------- W4_LAYOUT_GEMM
// Rows padded to a multiple of 128 (one MMA tile of weight rows), K to a multiple of 128.
//   codes:  [Npad][Kpad/2] bytes, row-major (TMA-loadable as a 2-D tensor). Inside every
//           32-bit word (8 consecutive k) the nibble slot p (bits [4p, 4p+4)) holds
//           q[k0 + p/2 + 4*(p%2)], so that w & 0x0F0F0F0F gives the bytes of k0..k0+3 and
//           (w >> 4) & 0x0F0F0F0F the bytes of k0+4..k0+7.
//   scales: [J = Kpad/g][Npad] u32 (group-major: one group's scales for consecutive rows are
//           contiguous), lo 16 bits fp16 scale, hi 16 bits zero (8 for symmetric).
//   zop:    [Npad][KZ] bf16 with Jr = K/g real groups and KZ = 3 Jr rounded up to 32: the
//           zero-point operand of the GEMM, a function of the scales and zeros above (kept
//           here so that the GEMM loads it by TMA). With v = s[n,j] * z[n,j] in fp32,
//           hi = bf16(v), lo = bf16(v - hi), row n holds
//           [hi(0..Jr-1) | hi(0..Jr-1) | lo(0..Jr-1) | 0 ...]; padding rows are 0.
struct GemmLayout {
    int64_t N, K, Npad, Kpad, J, Jr, KZ;
    int g;
    size_t codes_bytes, scales_bytes, zop_bytes, total;
};

// bf16 columns of a zero-point (or group-sum) operand row for Jr groups
inline int64_t zop_cols(int64_t Jr) { return (3 * Jr + 31) / 32 * 32; }

inline GemmLayout gemm_layout(int64_t N, int64_t K, int g) {
    GemmLayout L;
    L.N = N; L.K = K; L.g = g;
    L.Npad = (N + 127) / 128 * 128;
    L.Kpad = (K + 127) / 128 * 128;
    L.J = L.Kpad / g;
    L.Jr = K / g;
    L.KZ = zop_cols(L.Jr);
    L.codes_bytes = (size_t)L.Npad * (size_t)L.Kpad / 2;
    L.scales_bytes = (size_t)L.J * (size_t)L.Npad * 4;
    L.zop_bytes = (size_t)L.Npad * (size_t)L.KZ * 2;
    L.total = L.codes_bytes + L.scales_bytes + L.zop_bytes;
    return L;
}

}  // namespace w4
