// Host-side constant tables of the library: the NF4 codebook, its decision
// thresholds, and the bin table the quantize kernel uses to find the nearest
// code with one comparison.
#pragma once

#include <cstdint>

namespace qlora {

// Bin mapping used by the quantize kernel: x = fmaf(v, kBinMul, kBinAdd) is
// 1.5 * 2^23 + 64 + r with r = v * 63.5 rounded to the nearest integer (one
// rounding, ties to even; |r| <= 64 for v in [-1 - 2^-19, 1 + 2^-19]), so the
// low byte of x's bit pattern is u = 64 + r in [0, 128], and bin = u >> 2 (the
// byte offset of the bin's entry in a table of 4-byte entries is u & 0xFC).
constexpr float kBinMul = 63.5f;
constexpr float kBinAdd = 12582976.0f;  // 1.5 * 2^23 + 64, exact in fp32
constexpr int kBins = 33;

struct BinEntry {
  float threshold;  // T_j
  uint32_t j;       // code = j + (v >= T_j)
};

struct QuantTables {
  float codebook[16];     // ascending NF4 values, fp32
  float thresholds[15];   // T_i = smallest fp32 above the midpoint of codes i, i+1
  BinEntry bins[kBins];
};

// 4-bit data types: the NF4 codebook (default) and the FP4 comparison variant.
constexpr int kDtypeNf4 = 0;
constexpr int kDtypeFp4 = 1;

// Computed once on first use (thread-safe static initialisation).
const QuantTables& quant_tables(int dtype = kDtypeNf4);

}  // namespace qlora
