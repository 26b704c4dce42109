// Exhaustive host check of the quantize kernel's binning rule, for the NF4 and
// the FP4 tables: for every fp32 v in [-1 - 2^-19, 1 + 2^-19], the code the
// kernel forms from its bin table,
//   x = fmaf(v, kBinMul, kBinAdd), entry = bins[(bits(x) & 0xFC) >> 2],
//   code = (entry.j + 1) - [RN(v - entry.threshold) < 0],
// must equal the number of decision thresholds T_i with v >= T_i (the nearest
// code, ties to the lower index). Exit status 0 iff no value disagrees.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <thread>
#include <vector>

#include "host_tables.h"

using namespace qlora;

static uint64_t check_range(uint32_t lo, uint32_t hi, int sign, int dtype) {
  const QuantTables& t = quant_tables(dtype);
  uint64_t bad = 0;
  for (uint32_t bits = lo; bits < hi; ++bits) {
    const uint32_t b = bits | (sign ? 0x80000000u : 0u);
    float v;
    std::memcpy(&v, &b, 4);
    int ref = 0;
    for (int i = 0; i < 15; ++i) ref += (v >= t.thresholds[i]) ? 1 : 0;
    const float x = std::fmaf(v, kBinMul, kBinAdd);
    uint32_t xb;
    std::memcpy(&xb, &x, 4);
    const BinEntry& e = t.bins[(xb & 0xFCu) >> 2];
    const float d = v - e.threshold;
    uint32_t db;
    std::memcpy(&db, &d, 4);
    const int code = static_cast<int>(e.j + 1) - static_cast<int>(db >> 31);
    if (code != ref) {
      if (bad < 3) std::printf("mismatch: v=%a expected %d got %d\n", v, ref, code);
      ++bad;
    }
  }
  return bad;
}

int main() {
  // every bit pattern of [+0, 1 + 2^-19]: the quantize kernel's fast path feeds
  // the rule RN(w * rcp.approx(m)), which can exceed 1 by less than 2^-22
  const uint32_t end = 0x3F800011u;
  const unsigned nt = std::thread::hardware_concurrency() ? std::thread::hardware_concurrency() : 4;
  uint64_t total = 0;
  for (int dtype : {kDtypeNf4, kDtypeFp4}) {
    std::vector<std::thread> th;
    std::vector<uint64_t> bad(2 * nt, 0);
    for (int sign = 0; sign < 2; ++sign)
      for (unsigned k = 0; k < nt; ++k) {
        const uint32_t lo = static_cast<uint32_t>(uint64_t(end) * k / nt);
        const uint32_t hi = static_cast<uint32_t>(uint64_t(end) * (k + 1) / nt);
        th.emplace_back([&, lo, hi, sign, k] { bad[sign * nt + k] = check_range(lo, hi, sign, dtype); });
      }
    for (auto& x : th) x.join();
    uint64_t sub = 0;
    for (uint64_t b : bad) sub += b;
    std::printf("dtype %d: checked %llu values, %llu mismatches\n", dtype, 2ull * end,
                static_cast<unsigned long long>(sub));
    total += sub;
  }
  std::printf("%llu mismatches\n", static_cast<unsigned long long>(total));
  return total == 0 ? 0 : 1;
}
