// Host-side launchers of the library's kernels (one per .cu file group).
// All take device pointers, enqueue on `stream` and return cudaGetLastError().
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace qlora {

constexpr int kQuantBinWords = 257;  // 256 exponent bins + 1 CTA ticket (u64 each)

cudaError_t launch_quantize(const void* W, int64_t numel, uint8_t* packed, int8_t* absmax_q, float* dq_scale,
                            float* mean, float* absmax_scratch, unsigned long long* bins, int num_sms,
                            cudaStream_t stream);

cudaError_t launch_dequantize(const uint8_t* packed, const int8_t* absmax_q, const float* dq_scale,
                              const float* mean, void* out, int64_t numel, const float codebook[16],
                              int num_sms, cudaStream_t stream);

// Weight view used by the fused GEMM kernels.
struct Nf4View {
  const uint8_t* packed;
  const int8_t* absmax_q;
  const float* dq_scale;
  const float* mean;
  int64_t N;  // rows
  int64_t K;  // cols
};

// ---- LoRA skinny contractions (lora.cu) ----
// T[M,r] = X[M,K] A[r,K]^T (fp32); optionally sT[M,rpad] = bf16(s*T) with zero padding.
cudaError_t launch_lora_down(const void* X, const void* A, int64_t M, int64_t K, int r, float s, float* T,
                             void* sT_bf16, int rpad, int num_sms, cudaStream_t stream);
// U[M,r] = dY[M,N] B[N,r] (fp32) and sU[M,rpad] = bf16(s*U) (zero padded).
cudaError_t launch_lora_up_t(const void* dY, const void* B, int64_t M, int64_t N, int r, float s, float* U,
                             void* sU_bf16, int rpad, int num_sms, cudaStream_t stream);
// G[R,C] = s * P[M,R]^T Q[M,C], P fp32 (split hi/lo bf16 on the fly), Q bf16, reduced over M.
// Used for dA (P = U, Q = X) and dB (P = dY as bf16... see lora.cu).
cudaError_t launch_lora_grad_a(const float* U, const void* X, int64_t M, int64_t K, int r, float s, void* dA,
                               float* partial, int64_t partial_elems, int num_sms, cudaStream_t stream);
cudaError_t launch_lora_grad_b(const void* dY, const float* T, int64_t M, int64_t N, int r, float s, void* dB,
                               float* partial, int64_t partial_elems, int num_sms, cudaStream_t stream);
size_t lora_grad_partial_elems(int64_t M, int64_t cols, int r, int num_sms);
cudaError_t launch_zero_bf16(void* p, int64_t n, cudaStream_t stream);

// ---- decode (M <= 16) fused dequant GEMM (decode.cu) ----
cudaError_t launch_decode_fwd(const Nf4View& w, const void* X, int64_t M, const float* T, const void* B, int r,
                              float s, void* Y, float* partial, int ksplit, const float codebook[16],
                              int num_sms, cudaStream_t stream);
int decode_ksplit(int64_t N, int64_t K, int num_sms);
size_t decode_partial_elems(int64_t M, int64_t N, int ksplit);

// ---- tcgen05 GEMM (gemm_tc.cu) ----
// C[M, Nc] = A1[M, K1] * op(B1) + A2[M, K2] * op(B2), bf16 in, fp32 accumulate, bf16 out.
// B1/B2 are K-major ([Nc, K]) when b_mn_major == 0, or MN-major ([K, Nc]) when 1.
struct TcGemmArgs {
  const void* A1; const void* B1; int64_t K1;
  const void* A2; const void* B2; int64_t K2; int64_t lda2; int64_t ldb2;  // slab (may be K2 == 0)
  void* C; int64_t M; int64_t Nc;
  int b_mn_major;
};
cudaError_t launch_tc_gemm(const TcGemmArgs& a, int num_sms, cudaStream_t stream);

}  // namespace qlora
