// C ABI entry points (include/qlora.h): argument checks, workspace layout and
// kernel dispatch. Nothing here allocates, frees or synchronizes, except
// qlora_device_error, which reads the device error word.
#include "qlora.h"

#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "host_tables.h"
#include "kernels.h"

namespace qlora {
__device__ int32_t g_device_error = 0;
}  // namespace qlora

namespace {

using namespace qlora;

constexpr size_t kAlign = 256;
constexpr int kRefSms = 148;  // B200
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct DeviceInfo {
  int num_sms;
};

qlora_status device_info(DeviceInfo* info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (major != 10) return QLORA_ERR_DEVICE;
  info->num_sms = sms;
  return QLORA_OK;
}

// Storage kinds: dq_blocksize == 256 is double-quantized (absmax_q, dq_scale,
// mean), dq_blocksize == 0 is single-level (absmax). kind: 0 either, 1 only
// double-quantized, 2 only single-level.
qlora_status check_weight(const qlora_nf4_weight* q, bool need_rows, int kind = 0) {
  if (!q) return QLORA_ERR_INVALID_ARG;
  if (q->rows < 0 || q->cols <= 0) return QLORA_ERR_INVALID_ARG;
  const bool single = q->dq_blocksize == 0;
  if (q->blocksize != 64 || (q->dq_blocksize != 256 && !single)) return QLORA_ERR_UNSUPPORTED;
  if ((kind == 1 && single) || (kind == 2 && !single)) return QLORA_ERR_UNSUPPORTED;
  if (q->cols % 64) return QLORA_ERR_UNSUPPORTED;
  if (q->rows > (int64_t(1) << 31) || q->cols > (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED;
  if (need_rows && q->rows == 0) return QLORA_ERR_INVALID_ARG;
  if (q->rows > 0) {
    if (single) {
      if (!q->packed || !q->absmax) return QLORA_ERR_INVALID_ARG;
      if (!aligned(q->packed, 16) || !aligned(q->absmax, 4)) return QLORA_ERR_ALIGNMENT;
    } else {
      if (!q->packed || !q->absmax_q || !q->dq_scale || !q->mean) return QLORA_ERR_INVALID_ARG;
      if (!aligned(q->packed, 16) || !aligned(q->absmax_q, 16) || !aligned(q->dq_scale, 4) ||
          !aligned(q->mean, 4))
        return QLORA_ERR_ALIGNMENT;
    }
  }
  return QLORA_OK;
}

// The kernels' view of a checked weight (absmax non-null marks single-level storage).
Nf4View view(const qlora_nf4_weight* q) {
  if (q->dq_blocksize == 0) return Nf4View{q->packed, nullptr, nullptr, nullptr, q->rows, q->cols, q->absmax};
  return Nf4View{q->packed, q->absmax_q, q->dq_scale, q->mean, q->rows, q->cols, nullptr};
}

qlora_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

// Workspace query / check shared by every call that needs scratch.
// Returns QLORA_OK with *launch == false for a pure size query.
qlora_status workspace_check(void* ws, size_t* ws_bytes, size_t need, bool* launch) {
  if (!ws_bytes) return QLORA_ERR_INVALID_ARG;
  if (!ws) {
    *ws_bytes = need;
    *launch = false;
    return QLORA_OK;
  }
  if (*ws_bytes < need) return QLORA_ERR_WORKSPACE;
  if (!aligned(ws, kAlign)) return QLORA_ERR_ALIGNMENT;
  *launch = true;
  return QLORA_OK;
}

qlora_status check_linear(const void* X, int64_t M, const void* A, const void* B, int32_t r, const void* out) {
  if (M < 0) return QLORA_ERR_INVALID_ARG;
  if (r < 8 || r > 256 || r % 8) return QLORA_ERR_UNSUPPORTED;
  if (!A || !B || (M > 0 && (!X || !out))) return QLORA_ERR_INVALID_ARG;
  if ((X && !aligned(X, 16)) || !aligned(A, 16) || !aligned(B, 16) || (out && !aligned(out, 16)))
    return QLORA_ERR_ALIGNMENT;
  if (M > (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED;
  return QLORA_OK;
}

float lora_scale(float alpha, int32_t r) { return alpha / static_cast<float>(r); }

// Decode kernel choice, read on every call: QLORA_DECODE_RES=0 in the
// environment selects the TMA-ring kernel for every shape, =1 the X-resident
// kernel wherever it fits (for comparisons and tests); unset, the measured
// crossover decides.
// Training forward and dX with W' decoded inside the 2-CTA GEMMs
// (QLORA_FWD_FUSED=1) instead of a dequant launch and a GEMM over the
// dequantized copy; M >= 256.
bool fused_forward(int64_t M) {
  const char* e = std::getenv("QLORA_FWD_FUSED");
  return M >= 256 && e && e[0] == '1';
}

int res_mode() {
  const char* e = std::getenv("QLORA_DECODE_RES");
  if (e && e[0] == '0') return 0;
  if (e && e[0] == '1') return 1;
  return 2;
}

int32_t* device_error_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, qlora::g_device_error) != cudaSuccess) return nullptr;
  return static_cast<int32_t*>(p);
}

// Split count for the token reductions of dA / dB: enough units to cover the SMs.
int grad_splits(int64_t R, int rpad, int64_t M, int num_sms) {
  const int64_t tiles = ((R + 127) / 128) * (rpad / 64);
  if (tiles <= 0) return 1;
  const int64_t nkb = (M + 63) / 64;  // each k-block multiplies by the hi and lo halves together
  const int64_t sp = (2 * num_sms) / tiles;  // at most one round of the two resident CTAs per SM
  return split_count(nkb, static_cast<int>(sp < 1 ? 1 : sp));
}

// Split count for the K (or N) reduction of the rank-r products X A^T and dY B.
int red_splits(int64_t M, int rpad, int64_t Kred, int num_sms) {
  const int64_t tiles = ((M + 127) / 128) * (rpad / 64);
  if (tiles <= 0) return 1;
  const int64_t nkb = (Kred + 63) / 64;
  const int64_t sp = (2 * num_sms) / tiles;  // at most one round of the two resident CTAs per SM
  return split_count(nkb, static_cast<int>(sp < 1 ? 1 : sp));
}

// Workspace layout: consecutive 256-byte aligned regions.
struct Layout {
  size_t off = 0;
  size_t add(size_t bytes) {
    const size_t o = off;
    off += align_up(bytes);
    return o;
  }
  size_t total() const { return off > 0 ? off : kAlign; }
};

// Backward shared by qlora_linear_bwd (bf16 dA, dB), qlora_linear_bwd_f32 and
// qlora_linear_bwd_dp (fp32 dA, dB). The LoRA gradients are finished before the
// dX GEMM; `grads_ready`, when given, is recorded on the stream right after them.
qlora_status linear_bwd_impl(const qlora_nf4_weight* q, const void* X, int64_t M, const void* A, const void* B,
                             int32_t r, float alpha, const void* dY, const float* T_saved, void* dX, void* dA,
                             void* dB, bool f32, void* workspace, size_t* workspace_bytes, qlora_stream_t stream,
                             cudaEvent_t grads_ready = nullptr) {
  qlora_status st = check_weight(q, true);
  if (st != QLORA_OK) return st;
  if ((st = check_linear(X, M, A, B, r, dA)) != QLORA_OK) return st;
  if (!dA || !dB || (M > 0 && !dY)) return QLORA_ERR_INVALID_ARG;
  if (!aligned(dB, 16) || (dY && !aligned(dY, 16)) || (dX && !aligned(dX, 16))) return QLORA_ERR_ALIGNMENT;
  if (T_saved && !aligned(T_saved, 4)) return QLORA_ERR_ALIGNMENT;
  const int64_t N = q->rows, K = q->cols;
  if (N % 8) return QLORA_ERR_UNSUPPORTED;  // dY rows must be 16-byte multiples for the TMA tiles
  const int rpad = (r + 63) / 64 * 64;
  const float s = lora_scale(alpha, r);
  DeviceInfo di{kRefSms};
  const int splits_a = grad_splits(K, rpad, M, di.num_sms);
  const int splits_b = grad_splits(N, rpad, M, di.num_sms);
  Layout L;
  const size_t mp = static_cast<size_t>(M) * rpad * 2;
  const size_t off_wd = L.add(dX ? static_cast<size_t>(N) * K * 2 : 0);
  const size_t off_thi = L.add(mp), off_tlo = L.add(mp);
  const size_t off_su = L.add(mp), off_uhi = L.add(mp), off_ulo = L.add(mp);
  const size_t off_tail = L.add(dX ? kPairTailBytes : 0);
  const int splits_t = red_splits(M, rpad, K, di.num_sms);
  const int splits_u = red_splits(M, rpad, N, di.num_sms);
  size_t pmax = static_cast<size_t>(splits_a) * K * rpad;
  const size_t pb = static_cast<size_t>(splits_b) * N * rpad;
  const size_t pt = static_cast<size_t>(T_saved ? 0 : splits_t) * M * rpad;
  const size_t pu = static_cast<size_t>(splits_u) * M * rpad;
  if (pb > pmax) pmax = pb;
  if (pt > pmax) pmax = pt;
  if (pu > pmax) pmax = pu;
  const size_t off_p = L.add(pmax * sizeof(float));
  bool launch = false;
  st = workspace_check(workspace, workspace_bytes, L.total(), &launch);
  if (st != QLORA_OK || !launch) return st;
  if ((st = device_info(&di)) != QLORA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (M == 0) {
    if (f32) {
      cudaError_t e = cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * K * sizeof(float), cs);
      if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, static_cast<size_t>(N) * r * sizeof(float), cs);
      if (e == cudaSuccess && grads_ready) e = cudaEventRecord(grads_ready, cs);
      return cuda_status(e);
    }
    cudaError_t e = launch_zero_bf16(dA, static_cast<int64_t>(r) * K, di.num_sms, cs);
    if (e == cudaSuccess) e = launch_zero_bf16(dB, N * r, di.num_sms, cs);
    return cuda_status(e);
  }
  char* ws = static_cast<char*>(workspace);
  int32_t* err = device_error_word();
  const float* cb = quant_tables().codebook;
  void *Thi = ws + off_thi, *Tlo = ws + off_tlo, *sU = ws + off_su, *Uhi = ws + off_uhi, *Ulo = ws + off_ulo;
  float* P = reinterpret_cast<float*>(ws + off_p);
  cudaError_t e = cudaSuccess;
  // T = X A^T as a two-term bf16 split (from the saved fp32 T or recomputed)
  if (T_saved) {
    e = launch_split_hilo(T_saved, M, r, rpad, Thi, Tlo, di.num_sms, cs);
  } else {
    e = launch_gemm_lora_t(X, A, M, K, r, rpad, P, splits_t, di.num_sms, err, cs);
    if (e == cudaSuccess)
      e = launch_lora_finish(P, splits_t, M, r, rpad, s, nullptr, nullptr, Thi, Tlo, di.num_sms, cs);
  }
  // U = dY B: s U for the dX slab, U as hi + lo for dA
  if (e == cudaSuccess) e = launch_gemm_lora_u(dY, B, M, N, r, rpad, P, splits_u, di.num_sms, err, cs);
  if (e == cudaSuccess) e = launch_lora_finish(P, splits_u, M, r, rpad, s, nullptr, sU, Uhi, Ulo, di.num_sms, cs);
  // dA^T [K, r] = X^T U, reduced over tokens, then dA = s * (.)^T
  if (e == cudaSuccess) e = launch_gemm_lora_grad(X, K, Uhi, Ulo, M, rpad, P, splits_a, di.num_sms, err, cs);
  if (e == cudaSuccess) e = launch_grad_reduce(P, splits_a, K, rpad, r, s, true, dA, f32, di.num_sms, cs);
  // dB [N, r] = dY^T T
  if (e == cudaSuccess) e = launch_gemm_lora_grad(dY, N, Thi, Tlo, M, rpad, P, splits_b, di.num_sms, err, cs);
  if (e == cudaSuccess) e = launch_grad_reduce(P, splits_b, N, rpad, r, s, false, dB, f32, di.num_sms, cs);
  // the LoRA gradients are complete: a cross-rank sum may start while dX runs
  if (e == cudaSuccess && grads_ready) e = cudaEventRecord(grads_ready, cs);
  if (dX && fused_forward(M)) {  // W' decoded inside the GEMM
    if (e == cudaSuccess)
      e = launch_gemm_dx_nf4(dY, view(q), sU, A, M, r, rpad, dX, ws + off_tail, cb, di.num_sms, err, cs);
  } else if (dX) {
    void* Wd = ws + off_wd;
    if (e == cudaSuccess)
      e = launch_dequantize(view(q), Wd, cb, di.num_sms, cs);
    if (e == cudaSuccess)
      e = launch_gemm_dx(dY, Wd, sU, A, M, N, K, r, rpad, dX, ws + off_tail, di.num_sms, err, cs);
  }
  return cuda_status(e);
}

int dtype_index(qlora_dtype d) { return d == QLORA_DTYPE_FP4 ? kDtypeFp4 : kDtypeNf4; }

qlora_status quantize_single_impl(const void* W_bf16, const qlora_nf4_weight* q, int dtype, qlora_stream_t stream) {
  qlora_status st = check_weight(q, false, 2);
  if (st != QLORA_OK) return st;
  if (!W_bf16 && q->rows > 0) return QLORA_ERR_INVALID_ARG;
  if (W_bf16 && !aligned(W_bf16, 16)) return QLORA_ERR_ALIGNMENT;
  const int64_t numel = q->rows * q->cols;
  if (numel == 0) return QLORA_OK;
  DeviceInfo di;
  if ((st = device_info(&di)) != QLORA_OK) return st;
  return cuda_status(launch_quantize_single(W_bf16, numel, q->packed, q->absmax, di.num_sms,
                                            reinterpret_cast<cudaStream_t>(stream), dtype));
}

qlora_status quantize_dq_impl(const void* W_bf16, const qlora_nf4_weight* q, int dtype, void* workspace,
                              size_t* workspace_bytes, qlora_stream_t stream) {
  qlora_status st = check_weight(q, false, 1);
  if (st != QLORA_OK) return st;
  if (!W_bf16 && q->rows > 0) return QLORA_ERR_INVALID_ARG;
  if (W_bf16 && !aligned(W_bf16, 16)) return QLORA_ERR_ALIGNMENT;
  const int64_t numel = q->rows * q->cols;
  const int64_t nblk = numel / 64;
  const size_t off_absmax = align_up(kQuantScratchBytes);
  const size_t need = off_absmax + align_up(static_cast<size_t>(nblk) * sizeof(float));
  bool launch = false;
  st = workspace_check(workspace, workspace_bytes, need, &launch);
  if (st != QLORA_OK || !launch || numel == 0) return st;
  DeviceInfo di;
  if ((st = device_info(&di)) != QLORA_OK) return st;
  char* ws = static_cast<char*>(workspace);
  return cuda_status(launch_quantize(W_bf16, numel, q->packed, q->absmax_q, q->dq_scale, q->mean,
                                     reinterpret_cast<float*>(ws + off_absmax), ws, di.num_sms,
                                     reinterpret_cast<cudaStream_t>(stream), dtype));
}

qlora_status dequantize_impl(const qlora_nf4_weight* q, int dtype, void* out_bf16, qlora_stream_t stream) {
  qlora_status st = check_weight(q, false);
  if (st != QLORA_OK) return st;
  const int64_t numel = q->rows * q->cols;
  if (numel == 0) return QLORA_OK;
  if (!out_bf16) return QLORA_ERR_INVALID_ARG;
  if (!aligned(out_bf16, 16)) return QLORA_ERR_ALIGNMENT;
  DeviceInfo di;
  if ((st = device_info(&di)) != QLORA_OK) return st;
  return cuda_status(launch_dequantize(view(q), out_bf16, quant_tables(dtype).codebook, di.num_sms,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

// Forward shared by qlora_linear_fwd (one adapter, scale s = alpha / r) and
// qlora_linear_fwd_multi (col_scale: one scale per rank column, s = 1).
qlora_status linear_fwd_impl(const qlora_nf4_weight* q, const void* X, int64_t M, const void* A, const void* B,
                             int32_t r, float alpha, void* Y, float* T_save, void* workspace,
                             size_t* workspace_bytes, qlora_stream_t stream, const float* col_scale) {
  qlora_status st = check_weight(q, true);
  if (st != QLORA_OK) return st;
  if ((st = check_linear(X, M, A, B, r, Y)) != QLORA_OK) return st;
  if (T_save && !aligned(T_save, 4)) return QLORA_ERR_ALIGNMENT;
  const int64_t N = q->rows, K = q->cols;
  const int rpad = (r + 63) / 64 * 64;
  const float s = col_scale ? 1.0f : lora_scale(alpha, r);
  DeviceInfo di{kRefSms};  // split choices use the reference SM count so the size query needs no device
  const bool decode = M <= 16;
  // workspace layout
  Layout L;
  size_t off_T = 0, off_part = 0, off_cnt = 0, off_wd = 0, off_sT = 0, off_tail = 0;
  DecodePlan dplan{};
  ResPlan rplan{};
  if (decode) {
    dplan = decode_plan(M, N, K, kRefSms);
    const int mode = res_mode();
    rplan = M > 0 && mode != 0 ? res_plan(M, N, K, kRefSms, mode == 1) : ResPlan{};
    off_T = L.add(T_save ? 0 : static_cast<size_t>(M) * r * sizeof(float));
    off_part = L.add((rplan.ok ? res_partial_elems(rplan) : decode_partial_elems(dplan)) * sizeof(float));
    off_cnt = L.add((rplan.ok ? static_cast<size_t>(rplan.n_tiles) : decode_counter_words(dplan)) *
                    sizeof(unsigned int));
  } else {
    off_wd = L.add(static_cast<size_t>(N) * K * 2);
    off_sT = L.add(static_cast<size_t>(M) * rpad * 2);
    off_part = L.add(static_cast<size_t>(red_splits(M, rpad, K, di.num_sms)) * M * rpad * sizeof(float));
    off_tail = L.add(kPairTailBytes);
  }
  bool launch = false;
  st = workspace_check(workspace, workspace_bytes, L.total(), &launch);
  if (st != QLORA_OK || !launch || M == 0) return st;
  if ((st = device_info(&di)) != QLORA_OK) return st;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  int32_t* err = device_error_word();
  const float* cb = quant_tables().codebook;
  if (decode) {
    float* T = T_save ? T_save : reinterpret_cast<float*>(ws + off_T);
    return cuda_status(launch_decode_fwd(view(q), X, M, A, B, r, s, Y, T, reinterpret_cast<float*>(ws + off_part),
                                         reinterpret_cast<unsigned int*>(ws + off_cnt), dplan, rplan, cb, err, cs,
                                         col_scale));
  }
  void* Wd = ws + off_wd;
  void* sT = ws + off_sT;
  float* P = reinterpret_cast<float*>(ws + off_part);
  const int splits_t = red_splits(M, rpad, K, kRefSms);
  if (fused_forward(M)) {  // W' decoded inside the GEMM: no dequantized copy
    cudaError_t e = launch_gemm_lora_t(X, A, M, K, r, rpad, P, splits_t, di.num_sms, err, cs);
    if (e == cudaSuccess)
      e = launch_lora_finish(P, splits_t, M, r, rpad, s, T_save, sT, nullptr, nullptr, di.num_sms, cs, col_scale);
    if (e == cudaSuccess)
      e = launch_gemm_fwd_nf4(X, view(q), sT, B, M, r, rpad, Y, ws + off_tail, cb, di.num_sms, err, cs);
    return cuda_status(e);
  }
  cudaError_t e = launch_dequantize(view(q), Wd, cb, di.num_sms, cs);
  if (e == cudaSuccess) e = launch_gemm_lora_t(X, A, M, K, r, rpad, P, splits_t, di.num_sms, err, cs);
  if (e == cudaSuccess)
    e = launch_lora_finish(P, splits_t, M, r, rpad, s, T_save, sT, nullptr, nullptr, di.num_sms, cs, col_scale);
  if (e == cudaSuccess) e = launch_gemm_fwd(X, Wd, sT, B, M, N, K, r, rpad, Y, ws + off_tail, di.num_sms, err, cs);
  return cuda_status(e);
}

}  // namespace


extern "C" {

const char* qlora_status_string(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG";
    case QLORA_ERR_UNSUPPORTED: return "QLORA_ERR_UNSUPPORTED";
    case QLORA_ERR_ALIGNMENT: return "QLORA_ERR_ALIGNMENT";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA";
    case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE";
    case QLORA_ERR_DEVICE: return "QLORA_ERR_DEVICE";
  }
  return "QLORA_ERR_UNKNOWN";
}

qlora_status qlora_nf4_codebook(float out16[16]) {
  if (!out16) return QLORA_ERR_INVALID_ARG;
  std::memcpy(out16, quant_tables().codebook, sizeof(float) * 16);
  return QLORA_OK;
}

qlora_status qlora_nf4_storage_bytes(int64_t rows, int64_t cols, size_t out[4]) {
  if (!out || rows < 0 || cols < 0) return QLORA_ERR_INVALID_ARG;
  if (cols % 64) return QLORA_ERR_UNSUPPORTED;
  const int64_t numel = rows * cols;
  const int64_t nblk = numel / 64;
  out[0] = static_cast<size_t>(numel / 2);
  out[1] = static_cast<size_t>(nblk);
  out[2] = static_cast<size_t>((nblk + 255) / 256) * sizeof(float);
  out[3] = sizeof(float);
  return QLORA_OK;
}

qlora_status qlora_nf4_single_storage_bytes(int64_t rows, int64_t cols, size_t out[2]) {
  if (!out || rows < 0 || cols < 0) return QLORA_ERR_INVALID_ARG;
  if (cols % 64) return QLORA_ERR_UNSUPPORTED;
  const int64_t numel = rows * cols;
  out[0] = static_cast<size_t>(numel / 2);
  out[1] = static_cast<size_t>(numel / 64) * sizeof(float);
  return QLORA_OK;
}

qlora_status qlora_quantize_nf4(const void* W_bf16, const qlora_nf4_weight* q, qlora_stream_t stream) {
  return quantize_single_impl(W_bf16, q, kDtypeNf4, stream);
}

qlora_status qlora_quantize_nf4_dq(const void* W_bf16, const qlora_nf4_weight* q, void* workspace,
                                   size_t* workspace_bytes, qlora_stream_t stream) {
  return quantize_dq_impl(W_bf16, q, kDtypeNf4, workspace, workspace_bytes, stream);
}

qlora_status qlora_dequantize_nf4(const qlora_nf4_weight* q, void* out_bf16, qlora_stream_t stream) {
  return dequantize_impl(q, kDtypeNf4, out_bf16, stream);
}

qlora_status qlora_codebook(qlora_dtype dtype, float out16[16]) {
  if (!out16) return QLORA_ERR_INVALID_ARG;
  if (dtype != QLORA_DTYPE_NF4 && dtype != QLORA_DTYPE_FP4) return QLORA_ERR_UNSUPPORTED;
  std::memcpy(out16, quant_tables(dtype_index(dtype)).codebook, sizeof(float) * 16);
  return QLORA_OK;
}

qlora_status qlora_quantize_4bit(const void* W_bf16, const qlora_nf4_weight* q, qlora_dtype dtype, void* workspace,
                                 size_t* workspace_bytes, qlora_stream_t stream) {
  if (dtype != QLORA_DTYPE_NF4 && dtype != QLORA_DTYPE_FP4) return QLORA_ERR_UNSUPPORTED;
  if (!q) return QLORA_ERR_INVALID_ARG;
  if (q->dq_blocksize == 0) {  // single level: no workspace
    if (!workspace_bytes) return QLORA_ERR_INVALID_ARG;
    if (!workspace) {
      *workspace_bytes = kAlign;
      qlora_status st = check_weight(q, false, 2);
      return st;
    }
    return quantize_single_impl(W_bf16, q, dtype_index(dtype), stream);
  }
  return quantize_dq_impl(W_bf16, q, dtype_index(dtype), workspace, workspace_bytes, stream);
}

qlora_status qlora_dequantize_4bit(const qlora_nf4_weight* q, qlora_dtype dtype, void* out_bf16,
                                   qlora_stream_t stream) {
  if (dtype != QLORA_DTYPE_NF4 && dtype != QLORA_DTYPE_FP4) return QLORA_ERR_UNSUPPORTED;
  return dequantize_impl(q, dtype_index(dtype), out_bf16, stream);
}

qlora_status qlora_dequantize_nf4_dq(const qlora_nf4_weight* q, void* out_bf16, qlora_stream_t stream) {
  return qlora_dequantize_nf4(q, out_bf16, stream);
}

qlora_status qlora_linear_fwd(const qlora_nf4_weight* q, const void* X, int64_t M, const void* A,
                              const void* B, int32_t r, float alpha, void* Y, float* T_save, void* workspace,
                              size_t* workspace_bytes, qlora_stream_t stream) {
  return linear_fwd_impl(q, X, M, A, B, r, alpha, Y, T_save, workspace, workspace_bytes, stream, nullptr);
}

qlora_status qlora_linear_fwd_multi(const qlora_nf4_weight* q, const void* X, int64_t M, const void* A_cat,
                                    const void* B_cat, int32_t r_total, const float* col_scale, void* Y,
                                    void* workspace, size_t* workspace_bytes, qlora_stream_t stream) {
  if (!col_scale) return QLORA_ERR_INVALID_ARG;
  if (!aligned(col_scale, 4)) return QLORA_ERR_ALIGNMENT;
  return linear_fwd_impl(q, X, M, A_cat, B_cat, r_total, 1.0f, Y, nullptr, workspace, workspace_bytes, stream,
                         col_scale);
}

qlora_status qlora_pack_adapters(const qlora_lora_adapter* adapters, int32_t n_adapters, int64_t rows, int64_t cols,
                                 void* A_cat, void* B_cat, float* col_scale, qlora_stream_t stream) {
  if (n_adapters < 1 || !adapters || rows <= 0 || cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (n_adapters > kMaxMergeAdapters) return QLORA_ERR_UNSUPPORTED;
  if (!A_cat || !B_cat || !col_scale) return QLORA_ERR_INVALID_ARG;
  if (!aligned(A_cat, 16) || !aligned(B_cat, 16) || !aligned(col_scale, 4)) return QLORA_ERR_ALIGNMENT;
  MergeAdapter ma[kMaxMergeAdapters];
  int rt = 0;
  for (int a = 0; a < n_adapters; ++a) {
    const qlora_lora_adapter& ad = adapters[a];
    if (ad.r < 8 || ad.r > 256 || ad.r % 8) return QLORA_ERR_UNSUPPORTED;
    if (!ad.A || !ad.B) return QLORA_ERR_INVALID_ARG;
    if (!aligned(ad.A, 16) || !aligned(ad.B, 16)) return QLORA_ERR_ALIGNMENT;
    ma[a].A = ad.A;
    ma[a].B = ad.B;
    ma[a].r = ad.r;
    ma[a].c = ad.weight * lora_scale(ad.alpha, ad.r);  // fp32(w * s), as in qlora_merge_lora
    rt += ad.r;
  }
  if (rt > 256) return QLORA_ERR_UNSUPPORTED;
  DeviceInfo di;
  qlora_status st = device_info(&di);
  if (st != QLORA_OK) return st;
  return cuda_status(launch_pack_adapters(ma, n_adapters, rows, cols, A_cat, B_cat, col_scale, di.num_sms,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status qlora_linear_bwd(const qlora_nf4_weight* q, const void* X, int64_t M, const void* A,
                              const void* B, int32_t r, float alpha, const void* dY, const float* T_saved,
                              void* dX, void* dA, void* dB, void* workspace, size_t* workspace_bytes,
                              qlora_stream_t stream) {
  return linear_bwd_impl(q, X, M, A, B, r, alpha, dY, T_saved, dX, dA, dB, false, workspace, workspace_bytes,
                         stream);
}

qlora_status qlora_linear_bwd_f32(const qlora_nf4_weight* q, const void* X, int64_t M, const void* A,
                                  const void* B, int32_t r, float alpha, const void* dY, const float* T_saved,
                                  void* dX, float* dA, float* dB, void* workspace, size_t* workspace_bytes,
                                  qlora_stream_t stream) {
  return linear_bwd_impl(q, X, M, A, B, r, alpha, dY, T_saved, dX, dA, dB, true, workspace, workspace_bytes,
                         stream);
}

qlora_status qlora_linear_bwd_dp(const qlora_nf4_weight* q, const void* X, int64_t M, const void* A,
                                 const void* B, int32_t r, float alpha, const void* dY, const float* T_saved,
                                 void* dX, float* grads, qlora_event_t grads_ready, void* workspace,
                                 size_t* workspace_bytes, qlora_stream_t stream) {
  if (!q || !grads) return QLORA_ERR_INVALID_ARG;
  if (!aligned(grads, 16)) return QLORA_ERR_ALIGNMENT;
  // dA [r, K] then dB [N, r]; r % 8 == 0 keeps dB's start 16-byte aligned
  float* dB = grads + static_cast<int64_t>(r) * q->cols;
  return linear_bwd_impl(q, X, M, A, B, r, alpha, dY, T_saved, dX, grads, dB, true, workspace, workspace_bytes,
                         stream, reinterpret_cast<cudaEvent_t>(grads_ready));
}

qlora_status qlora_round_bf16(const float* src, void* dst_bf16, int64_t n, qlora_stream_t stream) {
  if (n < 0) return QLORA_ERR_INVALID_ARG;
  if (n == 0) return QLORA_OK;
  if (!src || !dst_bf16) return QLORA_ERR_INVALID_ARG;
  if (!aligned(src, 4) || !aligned(dst_bf16, 2)) return QLORA_ERR_ALIGNMENT;
  DeviceInfo di;
  qlora_status st = device_info(&di);
  if (st != QLORA_OK) return st;
  return cuda_status(launch_round_bf16(src, dst_bf16, n, di.num_sms, reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status qlora_merge_lora(const qlora_nf4_weight* q, const qlora_lora_adapter* adapters,
                              int32_t n_adapters, void* W_out, qlora_stream_t stream) {
  qlora_status st = check_weight(q, false);
  if (st != QLORA_OK) return st;
  if (n_adapters < 0 || (n_adapters > 0 && !adapters)) return QLORA_ERR_INVALID_ARG;
  if (n_adapters > kMaxMergeAdapters) return QLORA_ERR_UNSUPPORTED;
  MergeAdapter ma[kMaxMergeAdapters];
  for (int a = 0; a < n_adapters; ++a) {
    const qlora_lora_adapter& ad = adapters[a];
    if (ad.r < 8 || ad.r > 256 || ad.r % 8) return QLORA_ERR_UNSUPPORTED;
    if (!ad.A || !ad.B) return QLORA_ERR_INVALID_ARG;
    if (!aligned(ad.A, 16) || !aligned(ad.B, 16)) return QLORA_ERR_ALIGNMENT;
    ma[a].A = ad.A;
    ma[a].B = ad.B;
    ma[a].r = ad.r;
    ma[a].c = ad.weight * lora_scale(ad.alpha, ad.r);  // fp32(w * s)
  }
  const int64_t numel = q->rows * q->cols;
  if (numel == 0) return QLORA_OK;
  if (!W_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned(W_out, 16)) return QLORA_ERR_ALIGNMENT;
  if ((q->rows + 63) / 64 > 65535) return QLORA_ERR_UNSUPPORTED;
  DeviceInfo di;
  if ((st = device_info(&di)) != QLORA_OK) return st;
  return cuda_status(launch_merge(view(q), ma, n_adapters, W_out, quant_tables().codebook, di.num_sms,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status qlora_device_error(int32_t* code, qlora_stream_t stream) {
  if (!code) return QLORA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return QLORA_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, qlora::g_device_error, sizeof(v)) != cudaSuccess) return QLORA_ERR_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpyToSymbol(qlora::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return QLORA_ERR_CUDA;
  *code = v;
  return QLORA_OK;
}

}  // extern "C"
