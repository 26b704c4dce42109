// Host-side launchers of the library's kernels. All take device pointers,
// enqueue on `stream` and return the launch status (cudaGetLastError()).
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace qlora {

// Raises a kernel's dynamic shared memory limit once per device, safely from
// several host threads: one flag bit per device ordinal (for ordinals above 63
// the attribute is set on every call).
template <auto Kern>
cudaError_t ensure_smem_limit(int bytes) {
  static std::atomic<unsigned long long> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Quantize scratch besides the fp32 absmax: the 256 exponent-bin totals (u64)
// of the exact sum of the constants (the part a row shard's caller exchanges).
constexpr size_t kQuantScratchBytes = 256 * sizeof(unsigned long long);

// Number of non-empty pieces when `nkb` k-blocks are cut into pieces of
// ceil(nkb / want) blocks. The split-reduction GEMMs and the kernels that sum
// their partials must both use this count.
inline int split_count(int64_t nkb, int want) {
  if (nkb <= 0) return 1;
  if (want < 1) want = 1;
  if (want > nkb) want = static_cast<int>(nkb);
  const int64_t per = (nkb + want - 1) / want;
  return static_cast<int>((nkb + per - 1) / per);
}

// ---- quantize.cu / dequant.cu ----
// dtype: the 4-bit codebook (kDtypeNf4, or kDtypeFp4 of host_tables.h).
cudaError_t launch_quantize(const void* W, int64_t numel, uint8_t* packed, int8_t* absmax_q, float* dq_scale,
                            float* mean, float* absmax_scratch, void* totals_scratch, int num_sms,
                            cudaStream_t stream, int dtype = 0);

// The two halves of launch_quantize, for a weight quantized in row shards:
// first, the codes, the fp32 constants and the 256 exact bin totals of their
// sum (zeroed and then added into); second, after the totals of all shards have
// been summed, the mean over nblk_mean constants and the int8 codes and group
// scales of this shard's nblk constants.
cudaError_t launch_quantize_first(const void* W, int64_t nblk, uint8_t* packed, float* absmax_scratch,
                                  unsigned long long* totals, int num_sms, cudaStream_t stream, int dtype = 0);
cudaError_t launch_quantize_second(const float* absmax_scratch, int64_t nblk, const unsigned long long* totals,
                                   int64_t nblk_mean, int8_t* absmax_q, float* dq_scale, float* mean,
                                   int num_sms, cudaStream_t stream);

// Single-level storage: the codes and the fp32 block constants m_b only (pass 1).
cudaError_t launch_quantize_single(const void* W, int64_t numel, uint8_t* packed, float* absmax, int num_sms,
                                   cudaStream_t stream, int dtype = 0);

// A stored weight. Double-quantized: absmax_q, dq_scale and mean give the block
// constant m'_b = fmaf(absmax_q[b], dq_scale[b / 256], mean) and absmax is null.
// Single-level: absmax[b] is the constant itself and the other three are null.
struct Nf4View {
  const uint8_t* packed;
  const int8_t* absmax_q;
  const float* dq_scale;
  const float* mean;
  int64_t N;  // rows
  int64_t K;  // cols
  const float* absmax;
};

cudaError_t launch_dequantize(const Nf4View& w, void* out, const float codebook[16], int num_sms,
                              cudaStream_t stream);

// ---- decode.cu: M <= 16 forward ----
// Work split of the decode kernel: (128-row group, 256-wide K superblock)
// items cut into equal per-CTA ranges; fixed by (M, N, K) and a reference SM
// count.
struct DecodePlan {
  int mt;             // token tiles of 8 (1: M <= 8, 2: M <= 16)
  int64_t n_groups;   // ceil(N / 128)
  int64_t row_tiles;  // 16-row tiles: 8 * n_groups
  int64_t nsb;        // ceil(K / 256)
  int64_t n_items;    // n_groups * nsb
  int grid;           // CTAs = work ranges: min(n_items, CTA capacity)
  int max_seg;        // most CTAs sharing one row group
};
DecodePlan decode_plan(int64_t M, int64_t N, int64_t K, int ref_sms);
size_t decode_partial_elems(const DecodePlan& p);
size_t decode_counter_words(const DecodePlan& p);
// Plan of the X-resident decode kernel (decode_res.cu): token values held in
// shared memory, warp-level item ranges. ok is false when it does not fit.
struct ResPlan {
  bool ok;
  int mt;
  int64_t n_tiles;     // 16-row tiles
  int64_t n_items;     // n_tiles * ceil(K / 256)
  int64_t n_units;     // warps of the grid
  int grid;            // CTAs (one per SM)
  int x_stride;        // bytes per token row of the shared X copy
  int p_max;           // reduction slots per warp
  int cta_tiles;       // tile counters per CTA
  int max_cta_seg;     // most CTAs holding pieces of one tile
  size_t smem;         // dynamic shared memory per CTA
};
// force: use it wherever it fits, not only where it measured faster.
ResPlan res_plan(int64_t M, int64_t N, int64_t K, int num_sms, bool force = false);
size_t res_partial_elems(const ResPlan& p);
cudaError_t launch_decode_res_main(const Nf4View& w, const void* X, int64_t M, const void* B, int r, float s,
                                   void* Y, const float* T, float* partial, unsigned int* counters,
                                   const ResPlan& rp, const float codebook[16], cudaStream_t stream);

// T [M, r] fp32 receives X A^T; partial [decode_partial_elems] fp32 and
// counters [decode_counter_words] are scratch. With rp.ok the X-resident kernel
// runs (partial then holds res_partial_elems(rp) floats, counters rp.n_tiles words).
cudaError_t launch_decode_fwd(const Nf4View& w, const void* X, int64_t M, const void* A, const void* B, int r,
                              float s, void* Y, float* T, float* partial, unsigned int* counters,
                              const DecodePlan& p, const ResPlan& rp, const float codebook[16], int32_t* err,
                              cudaStream_t stream, const float* col_scale = nullptr);
// col_scale (fp32 [r] or null): T's column j is multiplied by col_scale[j] as it
// is formed (several adapters concatenated along r, each with its own scale);
// the caller then passes s = 1.

// ---- merge.cu: weighted LoRA adapters merged into the dequantized base ----
constexpr int kMaxMergeAdapters = 8;
struct MergeAdapter {
  const void* A;  // bf16 [r, K]
  const void* B;  // bf16 [N, r]
  int r;
  float c;        // fp32(weight * s)
};
// out (bf16 [N, K]) = bf16_rn(W' + sum_a c_a B_a A_a), sums in fp64 (order in merge.cu).
cudaError_t launch_merge(const Nf4View& w, const MergeAdapter* adapters, int n_adapters, void* out,
                         const float codebook[16], int num_sms, cudaStream_t stream);

// ---- gemm_tc.cu: tcgen05 GEMMs ----
// Scratch of the 2-CTA GEMMs for the tiles of a last wave split in two along K:
// at most kPairMaxTail such tiles, each with two fp32 halves of 256 x 256 and
// eight 64-bit flags. `tail_ws` (kPairTailBytes, 256-byte aligned) may be null:
// the tail is then not split.
constexpr int kPairMaxTail = 37;
constexpr size_t kPairTailBytes =
    static_cast<size_t>(kPairMaxTail) * (2 * 2 * 128 * 256 * sizeof(float) + 8 * sizeof(unsigned long long));
cudaError_t launch_gemm_fwd(const void* X, const void* Wd, const void* sT, const void* Bl, int64_t M, int64_t N,
                            int64_t K, int r, int rpad, void* Y, void* tail_ws, int num_sms, int32_t* err,
                            cudaStream_t stream);
// The same forward with W' decoded from the NF4 storage inside the GEMM (no
// dequantized copy of W' in memory); M >= 256.
cudaError_t launch_gemm_fwd_nf4(const void* X, const Nf4View& w, const void* sT, const void* Bl, int64_t M, int r,
                                int rpad, void* Y, void* tail_ws, const float codebook[16], int num_sms, int32_t* err,
                                cudaStream_t stream);
// dX with W' decoded inside the GEMM; M >= 256.
cudaError_t launch_gemm_dx_nf4(const void* dY, const Nf4View& w, const void* sU, const void* Al, int64_t M, int r,
                               int rpad, void* dX, void* tail_ws, const float codebook[16], int num_sms, int32_t* err,
                               cudaStream_t stream);
cudaError_t launch_gemm_dx(const void* dY, const void* Wd, const void* sU, const void* Al, int64_t M, int64_t N,
                           int64_t K, int r, int rpad, void* dX, void* tail_ws, int num_sms, int32_t* err,
                           cudaStream_t stream);
// Split-reduction partials P[splits][M][rpad] of X A^T (lora_t) and dY B (lora_u);
// launch_lora_finish sums them and writes the fp32 / scaled / hi+lo operands.
cudaError_t launch_gemm_lora_t(const void* X, const void* Al, int64_t M, int64_t K, int r, int rpad, float* P,
                               int splits, int num_sms, int32_t* err, cudaStream_t stream);
cudaError_t launch_gemm_lora_u(const void* dY, const void* Bl, int64_t M, int64_t N, int r, int rpad, float* P,
                               int splits, int num_sms, int32_t* err, cudaStream_t stream);
cudaError_t launch_gemm_lora_grad(const void* Q, int64_t R, const void* hi, const void* lo, int64_t M, int rpad,
                                  float* P, int splits, int num_sms, int32_t* err, cudaStream_t stream);

// ---- lora_misc.cu ----
cudaError_t launch_split_hilo(const float* T, int64_t M, int r, int rpad, void* hi, void* lo, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_lora_finish(const float* P, int splits, int64_t M, int r, int rpad, float s, float* f32,
                               void* s_bf16, void* hi, void* lo, int num_sms, cudaStream_t stream,
                               const float* col_scale = nullptr);
// Several adapters concatenated along r: A_cat [sum r_a, K] (the A_a one after
// another), B_cat [N, sum r_a] (the B_a side by side) and col_scale[j] = c_a of
// the adapter of column j, from the adapters' A, B and c.
cudaError_t launch_pack_adapters(const MergeAdapter* adapters, int n_adapters, int64_t N, int64_t K, void* A_cat,
                                 void* B_cat, float* col_scale, int num_sms, cudaStream_t stream);
cudaError_t launch_grad_reduce(const float* P, int splits, int64_t R, int rpad, int r, float s, bool transpose,
                               void* out, bool out_f32, int num_sms, cudaStream_t stream);
cudaError_t launch_zero_bf16(void* p, int64_t n, int num_sms, cudaStream_t stream);
// dst (bf16 [n]) = bf16_rn(src (fp32 [n])).
cudaError_t launch_round_bf16(const float* src, void* dst, int64_t n, int num_sms, cudaStream_t stream);

}  // namespace qlora
