// Kernel layouts of a prepacked INT4 weight (internal; the ABI treats them as opaque).
//
// Both layouts hold exactly the canonical codes, fp16 scales and int16 zeros, only moved:
// "Four-bit inference ... Tahoma", MSE clipping -- portable codes, scales and zero terms are
// rearranged once into a GPU-specific layout, without dequantizing or requantizing.
#pragma once
#include <stdint.h>
#include <stddef.h>

#ifdef __CUDACC__
#define W4_HD __host__ __device__
#else
#define W4_HD
#endif

namespace w4 {

// ---------------------------------------------------------------- W4_LAYOUT_GEMV
// One record per weight row, rows in order, so that any run of consecutive rows is one
// contiguous byte range (the GEMV stages whole rows with one bulk copy):
//   record n = [codes: K/2 bytes, the canonical bytes of row n (byte j = q[2j] | q[2j+1] << 4)]
//              [scales: J = K/g u32, lo 16 bits the fp16 scale, hi 16 bits the zero (8 for
//               symmetric weights), padded with zero words to a multiple of 16 bytes]
// so that, in every 32-bit code word (8 consecutive k), w & 0x0F0F0F0F holds the codes of
// the even k and w & 0xF0F0F0F0 sixteen times the codes of the odd k, byte by byte.
struct GemvLayout {
    int64_t N, K, J;
    int g;
    size_t code_bytes;   // per row
    size_t row_bytes;    // record size (multiple of 16)
    size_t total;
};

inline GemvLayout gemv_layout(int64_t N, int64_t K, int g) {
    GemvLayout L;
    L.N = N; L.K = K; L.g = g;
    L.J = K / g;
    L.code_bytes = (size_t)K / 2;
    L.row_bytes = L.code_bytes + ((size_t)L.J * 4 + 15) / 16 * 16;
    L.total = (size_t)N * L.row_bytes;
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

// ---------------------------------------------------------------- W4_LAYOUT_TC
// Units of 128 weight rows x KS k (KS = max(128, g)): tiles of 128 rows in order, inside a
// tile its k-blocks in order, so that any run of consecutive units is one contiguous byte
// range. Rows are padded to a multiple of 128 and K to a multiple of KS with zero codes and
// zero scales. One unit is one record:
//   [codes: KS/32 chunks x 128 rows x 16 bytes, chunk c of row r at byte (c * 128 + r) * 16;
//    inside every 32-bit word (8 consecutive k from k0) nibble p holds q[k0 + 2p] for p < 4
//    and q[k0 + 2(p - 4) + 1] for p >= 4, so that (w >> 4s) & 0x000F000F holds the codes of
//    k0 + 2s and k0 + 2s + 1 in its two 16-bit halves]
//   [scales: KS/g groups x 128 rows of u32 (group-major), lo 16 bits fp16 scale, hi 16 bits
//    zero (8 for symmetric weights)]
struct TcLayoutGeo {
    W4_HD static constexpr int ks(int g) { return g > 128 ? g : 128; }
    W4_HD static constexpr uint32_t code_bytes(int g) { return 128u * (uint32_t)ks(g) / 2u; }
    W4_HD static constexpr uint32_t record_bytes(int g) { return code_bytes(g) + (uint32_t)(ks(g) / g) * 128u * 4u; }
};

struct TcLayout {
    int64_t N, K, T, NKB;
    int g;
    size_t rec, total;
};

inline TcLayout tc_layout(int64_t N, int64_t K, int g) {
    TcLayout L;
    L.N = N; L.K = K; L.g = g;
    L.T = (N + 127) / 128;
    L.NKB = (K + TcLayoutGeo::ks(g) - 1) / TcLayoutGeo::ks(g);
    L.rec = TcLayoutGeo::record_bytes(g);
    L.total = (size_t)L.T * (size_t)L.NKB * L.rec;
    return L;
}

}  // namespace w4
