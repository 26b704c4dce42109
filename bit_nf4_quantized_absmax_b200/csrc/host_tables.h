// Host-side constant tables of the library: the NF4 codebook, its decision
// thresholds, and the bin table the quantize kernel uses to find the nearest
// code with one comparison.
#pragma once

#include <cstdint>

namespace qlora {

// Bin mapping used by the quantize kernel: x = fmaf(v, kBinScale, 3.0f) lies
// in [2, 4) for v in [-1, 1]; the top kBinBits mantissa bits of x index the bin.
constexpr float kBinScale = 0.9990234375f;  // 1 - 2^-10, exact in fp32
constexpr int kBinBits = 5;
constexpr int kBins = 1 << kBinBits;

struct BinEntry {
  float threshold;  // T_j
  uint32_t j;       // code = j + (v >= T_j)
};

struct QuantTables {
  float codebook[16];     // ascending NF4 values, fp32
  float thresholds[15];   // T_i = smallest fp32 above the midpoint of codes i, i+1
  BinEntry bins[kBins];
};

// Computed once on first use (thread-safe static initialisation).
const QuantTables& quant_tables();

}  // namespace qlora
