// Host-side constant tables of the library: the NF4 codebook, its decision
// thresholds, and the bin table the quantize kernel uses to find the nearest
// code with one comparison.
#pragma once

#include <cstdint>

namespace qlora {

// Bin mapping used by the quantize kernel: x = fmaf(v, kBinMul, kBinAdd) is
// 1.5 * 2^23 + 128 + r with r = v * 127 rounded to the nearest integer (one
// rounding; |r| <= 127 for v in [-1, 1]), so the low byte of x's bit pattern is
// u = 128 + r in [1, 255], and bin = u >> 3 (the byte offset of the bin's
// 8-byte table entry is u & 0xF8).
constexpr float kBinMul = 127.0f;
constexpr float kBinAdd = 12583040.0f;  // 1.5 * 2^23 + 128, exact in fp32
constexpr int kBins = 32;

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
