// NF4 (and FP4) codebooks and quantization tables, computed on the host.
//
// Codebook: normal quantiles at equally spaced probabilities ("Guanaco",
// "Technical Innovations": a 4-bit type for normally distributed weights;
// QLoRA errata page, paper p.5 Section 3: a discrete zero and all 2^k values
// used). 8 positive values Phi^-1(1/2 + (d - 1/2) j/8), 7 negative values
// -Phi^-1(1/2 + (d - 1/2) j/7), an exact zero, all divided by Phi^-1(d), with
// d = 1 - (1/30 + 1/32)/2. Phi^-1 is found by Newton's method on
// Phi(x) = erfc(-x/sqrt 2)/2, started at x = 0 (Phi is concave on x > 0, so
// the iterates increase monotonically to the root).
#include "host_tables.h"

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>

namespace qlora {
namespace {

double normal_quantile_upper(double p) {
  // p in (1/2, 1)
  const double inv_sqrt2 = 0.70710678118654752440;
  const double inv_sqrt2pi = 0.39894228040143267794;
  double x = 0.0;
  for (int it = 0; it < 200; ++it) {
    double f = 0.5 * std::erfc(-x * inv_sqrt2) - p;
    double d = inv_sqrt2pi * std::exp(-0.5 * x * x);
    double dx = f / d;
    double xn = x - dx;
    if (xn == x) break;
    x = xn;
    if (std::fabs(dx) <= 1e-17 * std::fmax(1.0, std::fabs(x))) break;
  }
  return x;
}

void nf4_values(double (&vals)[16]) {
  const double d = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
  const double top = normal_quantile_upper(d);
  int n = 0;
  for (int j = 7; j >= 1; --j) vals[n++] = -normal_quantile_upper(0.5 + (d - 0.5) * j / 7.0) / top;
  vals[n++] = 0.0;
  for (int j = 1; j <= 8; ++j) vals[n++] = normal_quantile_upper(0.5 + (d - 0.5) * j / 8.0) / top;
  // the end points are exactly -1 and +1 (p = d on both sides)
  vals[0] = -1.0;
  vals[15] = 1.0;
}

// FP4 ("Float4" of the QLoRA errata page's findings on the paper's p.8 Table 4,
// which compares it with NFloat4; the pages give no format). Reading: the 4-bit
// float with 1 sign, 2 exponent and 1 mantissa bit, magnitudes
// {0, 0.5, 1, 1.5, 2, 3, 4, 6}, divided by 6 so that the range is [-1, 1]. Its
// two zero encodings are one value, kept once: 15 distinct values in ascending
// order at indices 0..14, and index 15 repeats +1, so that no value ever maps
// to it (the nearest code takes the lower index on a tie).
void fp4_values(double (&vals)[16]) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  int n = 0;
  for (int k = 7; k >= 1; --k) vals[n++] = -mag[k] / 6.0;
  for (int k = 0; k < 8; ++k) vals[n++] = mag[k] / 6.0;
  vals[15] = 1.0;
}

void build(QuantTables& t, int dtype) {
  double vals[16];
  if (dtype == kDtypeFp4)
    fp4_values(vals);
  else
    nf4_values(vals);
  for (int i = 0; i < 16; ++i) t.codebook[i] = static_cast<float>(vals[i]);

  // Decision thresholds: nearest code with ties to the lower index means
  // code(v) = #{i : v > mid_i}, mid_i = (c_i + c_{i+1}) / 2 (exact in double).
  // For fp32 v that is #{i : v >= T_i} with T_i the smallest float above mid_i.
  // (A repeated last value, as in FP4, puts its threshold above 1: never reached.)
  for (int i = 0; i < 15; ++i) {
    double mid = 0.5 * (static_cast<double>(t.codebook[i]) + static_cast<double>(t.codebook[i + 1]));
    float f = static_cast<float>(mid);
    if (static_cast<double>(f) <= mid) f = std::nextafterf(f, 2.0f);
    t.thresholds[i] = f;
  }

  // Bin table. Bin b holds u = 64 + r in [4b, 4b + 3], r = round(v * 63.5) (ties
  // to even), so it can only see v with v * 63.5 in [4b - 64.5, 4b - 60.5];
  // widen by 2^-20 for margin. Each widened bin must contain at most one
  // threshold (bins are ~0.063 wide, thresholds >= 0.08 apart); checked below.
  const double P = static_cast<double>(kBinMul);
  for (int b = 0; b < kBins; ++b) {
    double lo = (4.0 * b - 64.5) / P - std::ldexp(1.0, -20);
    double hi = (4.0 * b - 60.5) / P + std::ldexp(1.0, -20);
    int inside = -1, count = 0, below = 0;
    for (int i = 0; i < 15; ++i) {
      double T = t.thresholds[i];
      if (T >= lo && T <= hi) { inside = i; ++count; }
      if (T < lo) ++below;
    }
    if (count > 1) {
      std::fprintf(stderr, "qlora: internal error, bin %d holds %d thresholds\n", b, count);
      std::abort();
    }
    uint32_t j;
    if (count == 1) {
      j = static_cast<uint32_t>(inside);            // below T_j: code j; at/above: j + 1
    } else if (below == 0) {
      j = 0;                                        // whole bin below T_0: code 0
    } else {
      j = static_cast<uint32_t>(below - 1);         // v >= T_{below-1} always: code below
    }
    t.bins[b].threshold = t.thresholds[j];
    t.bins[b].j = j;
  }
}

}  // namespace

const QuantTables& quant_tables(int dtype) {
  static const QuantTables nf4 = [] {
    QuantTables t;
    std::memset(&t, 0, sizeof(t));
    build(t, kDtypeNf4);
    return t;
  }();
  static const QuantTables fp4 = [] {
    QuantTables t;
    std::memset(&t, 0, sizeof(t));
    build(t, kDtypeFp4);
    return t;
  }();
  return dtype == kDtypeFp4 ? fp4 : nf4;
}

}  // namespace qlora
