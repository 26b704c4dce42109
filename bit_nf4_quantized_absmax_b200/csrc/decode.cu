// Decode-shaped QLoRA forward (M <= 16 tokens), bound by the bandwidth of the
// packed 4-bit weights ("QLoRA vs ChatGPT", capability 5: the frozen weight is
// dequantized on the fly, block by block).
//
// Y[M, N] = X W'^T + s T B^T with T = X A^T computed first (k_lora_t_small).
//
// k_decode computes D = W' X^T with the weight as the MMA's A operand
// (mma.sync m16n8k16, bf16 in, fp32 accumulate) so that the 16 weight rows fill
// the MMA's M dimension and the tokens its N dimension. The reduction index is
// permuted: over a 256-wide "superblock" lane (g, t) supplies k-slots
// {2t, 2t+1, 2t+8, 2t+9} of every one of the 16 MMAs from the 64 consecutive
// weights of block 4*sb + t of rows g and g+8, and the matching token values.
// Each lane therefore decodes whole 64-weight blocks: one 16-entry bf16 table
// per block (bit-identical to the standalone dequant) and byte-permute lookups.
// The K range of a row tile may be split across CTAs; the last CTA of a row
// tile (ticket counter, no waiting) sums the partials in a fixed order and
// applies the LoRA term.
#include "common.cuh"
#include "kernels.h"
#include "nf4_lut.cuh"

namespace qlora {
namespace {

constexpr int kDecodeWarps = 8;

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct RowBlock {
  uint4 n0, n1;   // 64 codes
  int qv;         // int8 block constant code
  float sc;       // its group scale (the decoded constant is formed when the block is used)
};

template <bool V8>
__device__ __forceinline__ RowBlock load_row_block(const uint8_t* __restrict__ packed, const int8_t* __restrict__ q,
                                                   const float* __restrict__ dqs, float mu, int64_t n,
                                                   int64_t nkb_row, int64_t kb, bool valid) {
  RowBlock rb;
  if (valid) {
    const int64_t blk = n * nkb_row + kb;
    const uint4* p = reinterpret_cast<const uint4*>(packed + blk * 32);
    if (V8) {
      uint32_t r[8];
      ld_global_cs_v8(p, r);
      rb.n0 = make_uint4(r[0], r[1], r[2], r[3]);
      rb.n1 = make_uint4(r[4], r[5], r[6], r[7]);
    } else {
      rb.n0 = __ldcs(p);
      rb.n1 = __ldcs(p + 1);
    }
    rb.qv = static_cast<int>(__ldg(q + blk));
    rb.sc = __ldg(dqs + (blk >> 8));
  } else {
    rb.n0 = make_uint4(0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u);
    rb.n1 = rb.n0;
    rb.qv = 0;
    rb.sc = 0.0f;
  }
  return rb;
}

__device__ __forceinline__ uint32_t nib_word(const RowBlock& rb, int w) {
  switch (w) {
    case 0: return rb.n0.x;
    case 1: return rb.n0.y;
    case 2: return rb.n0.z;
    case 3: return rb.n0.w;
    case 4: return rb.n1.x;
    case 5: return rb.n1.y;
    case 6: return rb.n1.z;
    default: return rb.n1.w;
  }
}

template <int MT, bool V8>
__global__ void __launch_bounds__(kDecodeWarps * 32, 2)
k_decode(const uint8_t* __restrict__ packed, const int8_t* __restrict__ q, const float* __restrict__ dqs,
         const float* __restrict__ mean, const __nv_bfloat16* __restrict__ X, int M, int64_t N, int64_t K,
         const float* __restrict__ T, const __nv_bfloat16* __restrict__ Bl, int r, float s,
         __nv_bfloat16* __restrict__ Y, float* __restrict__ partial, unsigned int* __restrict__ counters,
         int ksplit, int n_units, const __grid_constant__ Nf4Codebook cb) {
  __shared__ float red[kDecodeWarps][16][16];
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t nkb_row = K / 64;
  const int64_t nsb = (nkb_row + 3) / 4;
  const int64_t per = (nsb + ksplit - 1) / ksplit;
  const float mu = *mean;
  const int ntok = 8 * MT;
  bool t_ready = false;  // the LoRA-down kernel (T, ticket counters) has completed

  // Persistent loop over (16-row tile, K chunk) units.
  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const int64_t tile = unit / ksplit;
    const int split = unit % ksplit;
    const int64_t n0 = tile * 16;
    const int64_t sb_begin = split * per;
    const int64_t sb_end = min(nsb, sb_begin + per);
    const int64_t na = n0 + g, nb = n0 + g + 8;

    // two independent accumulator chains (even and odd MMA steps)
    float acc[2][MT][4];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int j = 0; j < MT; ++j) acc[c][j][0] = acc[c][j][1] = acc[c][j][2] = acc[c][j][3] = 0.0f;

    int64_t sb = sb_begin + warp;
    RowBlock na_next, nb_next;  // codes and block constants of the warp's next superblock
    if (sb < sb_end) {
      const int64_t kb = sb * 4 + t;
      const bool kv = kb < nkb_row;
      na_next = load_row_block<V8>(packed, q, dqs, mu, na, nkb_row, kb, kv && na < N);
      nb_next = load_row_block<V8>(packed, q, dqs, mu, nb, nkb_row, kb, kv && nb < N);
    }
    for (; sb < sb_end; sb += kDecodeWarps) {
      const int64_t kb = sb * 4 + t;
      const bool kv = kb < nkb_row;
      const RowBlock ra = na_next, rbk = nb_next;
      // token values for this lane's 64 k positions: tokens g (tile 0) and g + 8 (tile 1),
      // fetched 16 at a time (L1-resident; X is small)
      const uint4* xp[MT];
      bool xok[MT];
#pragma unroll
      for (int j = 0; j < MT; ++j) {
        const int tok = g + 8 * j;
        xok[j] = kv && tok < M;
        xp[j] = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(tok) * K + kb * 64);
      }
      const int64_t sbn = sb + kDecodeWarps;  // prefetch while this superblock is decoded
      if (sbn < sb_end) {
        const int64_t kbn = sbn * 4 + t;
        const bool kvn = kbn < nkb_row;
        na_next = load_row_block<V8>(packed, q, dqs, mu, na, nkb_row, kbn, kvn && na < N);
        nb_next = load_row_block<V8>(packed, q, dqs, mu, nb, nkb_row, kbn, kvn && nb < N);
      }
      const Nf4Lut la = make_nf4_lut(cb, __fmaf_rn(static_cast<float>(ra.qv), ra.sc, mu));
      const Nf4Lut lb = make_nf4_lut(cb, __fmaf_rn(static_cast<float>(rbk.qv), rbk.sc, mu));
      uint4 xv[MT][2];
#pragma unroll
      for (int st = 0; st < 16; ++st) {
        if ((st & 3) == 0) {
#pragma unroll
          for (int j = 0; j < MT; ++j) {
            if (!xok[j]) {
              xv[j][0] = xv[j][1] = make_uint4(0, 0, 0, 0);
            } else if (V8) {
              uint32_t rr[8];
              ld_global_nc_v8(xp[j] + (st >> 1), rr);
              xv[j][0] = make_uint4(rr[0], rr[1], rr[2], rr[3]);
              xv[j][1] = make_uint4(rr[4], rr[5], rr[6], rr[7]);
            } else {
              xv[j][0] = __ldg(xp[j] + (st >> 1));
              xv[j][1] = __ldg(xp[j] + (st >> 1) + 1);
            }
          }
        }
        const uint32_t wa = nib_word(ra, st >> 1) >> (16 * (st & 1));
        const uint32_t wb = nib_word(rbk, st >> 1) >> (16 * (st & 1));
        uint32_t a0, a1, a2, a3;
        nf4_lookup4(la, wa, a0, a2);   // row g: k-slots (2t, 2t+1) and (2t+8, 2t+9)
        nf4_lookup4(lb, wb, a1, a3);   // row g + 8
#pragma unroll
        for (int j = 0; j < MT; ++j) {
          const uint4 x4 = xv[j][(st >> 1) & 1];
          const uint32_t b0 = (st & 1) ? x4.z : x4.x;
          const uint32_t b1 = (st & 1) ? x4.w : x4.y;
          mma16816(acc[st & 1][j], a0, a1, a2, a3, b0, b1);
        }
      }
    }

    // acc[j]: (row g, token 8j + 2t), (g, 8j + 2t + 1), (g + 8, 8j + 2t), (g + 8, 8j + 2t + 1)
    __syncthreads();  // the previous unit's epilogue has finished reading red
#pragma unroll
    for (int j = 0; j < MT; ++j) {
      red[warp][g][8 * j + 2 * t] = acc[0][j][0] + acc[1][j][0];
      red[warp][g][8 * j + 2 * t + 1] = acc[0][j][1] + acc[1][j][1];
      red[warp][g + 8][8 * j + 2 * t] = acc[0][j][2] + acc[1][j][2];
      red[warp][g + 8][8 * j + 2 * t + 1] = acc[0][j][3] + acc[1][j][3];
    }
    __syncthreads();
    if (!t_ready) {  // T and the counters come from the preceding LoRA-down kernel
      pdl_enter();
      t_ready = true;
    }

    if (ksplit == 1) {
      for (int e = threadIdx.x; e < 16 * ntok; e += blockDim.x) {
        const int row = e / ntok, tok = e % ntok;
        const int64_t n = n0 + row;
        if (tok >= M || n >= N) continue;
        float y = 0.0f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) y += red[w][row][tok];
        float l = 0.0f;
        for (int jj = 0; jj < r; ++jj)
          l = fmaf(T[static_cast<int64_t>(tok) * r + jj], __bfloat162float(Bl[n * r + jj]), l);
        Y[static_cast<int64_t>(tok) * N + n] = __float2bfloat16_rn(fmaf(s, l, y));
      }
      continue;
    }

    // split K: publish this unit's partial, the last unit of the row tile finishes
    for (int e = threadIdx.x; e < 16 * ntok; e += blockDim.x) {
      const int row = e / ntok, tok = e % ntok;
      const int64_t n = n0 + row;
      if (tok >= M || n >= N) continue;
      float y = 0.0f;
#pragma unroll
      for (int w = 0; w < kDecodeWarps; ++w) y += red[w][row][tok];
      partial[(static_cast<int64_t>(split) * M + tok) * N + n] = y;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const unsigned int prev = atomicAdd(&counters[tile], 1u);
      s_last = (prev == static_cast<unsigned int>(ksplit - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (!s_last) continue;
    __threadfence();
    for (int e = threadIdx.x; e < 16 * ntok; e += blockDim.x) {
      const int row = e / ntok, tok = e % ntok;
      const int64_t n = n0 + row;
      if (tok >= M || n >= N) continue;
      float y = 0.0f;
      for (int sp = 0; sp < ksplit; ++sp) y += __ldcg(&partial[(static_cast<int64_t>(sp) * M + tok) * N + n]);
      float l = 0.0f;
      for (int jj = 0; jj < r; ++jj)
        l = fmaf(T[static_cast<int64_t>(tok) * r + jj], __bfloat162float(Bl[n * r + jj]), l);
      Y[static_cast<int64_t>(tok) * N + n] = __float2bfloat16_rn(fmaf(s, l, y));
    }
    if (threadIdx.x == 0) counters[tile] = 0u;
  }
  if (!t_ready) pdl_enter();
}

// T[m, j] = sum_k X[m, k] A[j, k] for M <= 16 (fp32 on CUDA cores), one CTA per
// adapter row j, 16-byte loads (8 k per thread and step). Block 0 also clears
// the decode kernel's ticket counters.
template <int MT>
__global__ void __launch_bounds__(256)
k_lora_t_small(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ A, int M, int64_t K, int r,
               float* __restrict__ T, unsigned int* __restrict__ counters, int n_counters) {
  __shared__ float red[8][8 * MT];
  pdl_enter();  // after this, the decode kernel may start its main loop
  const int j = blockIdx.x;
  if (j == 0)
    for (int i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0u;
  float acc[8 * MT];
#pragma unroll
  for (int m = 0; m < 8 * MT; ++m) acc[m] = 0.0f;
  const uint4* a4 = reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * K);
  for (int64_t k8 = threadIdx.x; k8 < K / 8; k8 += blockDim.x) {
    const uint4 av = __ldg(a4 + k8);
    const float a[8] = {bf16lo_to_f32(av.x), bf16hi_to_f32(av.x), bf16lo_to_f32(av.y), bf16hi_to_f32(av.y),
                        bf16lo_to_f32(av.z), bf16hi_to_f32(av.z), bf16lo_to_f32(av.w), bf16hi_to_f32(av.w)};
#pragma unroll
    for (int m = 0; m < 8 * MT; ++m) {
      if (m < M) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m) * K) + k8);
        float s = acc[m];
        s = fmaf(a[0], bf16lo_to_f32(xv.x), s);
        s = fmaf(a[1], bf16hi_to_f32(xv.x), s);
        s = fmaf(a[2], bf16lo_to_f32(xv.y), s);
        s = fmaf(a[3], bf16hi_to_f32(xv.y), s);
        s = fmaf(a[4], bf16lo_to_f32(xv.z), s);
        s = fmaf(a[5], bf16hi_to_f32(xv.z), s);
        s = fmaf(a[6], bf16lo_to_f32(xv.w), s);
        s = fmaf(a[7], bf16hi_to_f32(xv.w), s);
        acc[m] = s;
      }
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 0; m < 8 * MT; ++m) {
    float v = acc[m];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][m] = v;
  }
  __syncthreads();
  if (threadIdx.x < M) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[w][threadIdx.x];
    T[static_cast<int64_t>(threadIdx.x) * r + j] = v;
  }
}

}  // namespace

// K chunks per 16-row tile: each warp keeps two superblocks per unit when K
// allows it (so the next superblock's loads overlap the current one).
int decode_ksplit(int64_t N, int64_t K, int num_sms) {
  (void)N;
  (void)num_sms;
  const int64_t nsb = (K / 64 + 3) / 4;
  int64_t ks = nsb / (2 * kDecodeWarps);
  return static_cast<int>(ks < 1 ? 1 : ks);
}

size_t decode_partial_elems(int64_t M, int64_t N, int ksplit) {
  return ksplit > 1 ? static_cast<size_t>(ksplit) * M * N : 0;
}

size_t decode_counter_words(int64_t N) { return static_cast<size_t>((N + 15) / 16); }

cudaError_t launch_decode_fwd(const Nf4View& w, const void* X, int64_t M, const void* A, const void* B, int r,
                              float s, void* Y, float* T, float* partial, unsigned int* counters, int ksplit,
                              const float codebook[16], cudaStream_t stream) {
  Nf4Codebook cb;
  for (int i = 0; i < 16; ++i) cb.c[i] = codebook[i];
  const int64_t row_tiles = (w.N + 15) / 16;
  {
    cudaError_t e0 = launch_pdl(M <= 8 ? k_lora_t_small<1> : k_lora_t_small<2>, dim3(r), dim3(256), 0, stream,
                                reinterpret_cast<const __nv_bfloat16*>(X), reinterpret_cast<const __nv_bfloat16*>(A),
                                static_cast<int>(M), w.K, r, T, counters, static_cast<int>(row_tiles));
    if (e0 != cudaSuccess) return e0;
  }
  const int n_units = static_cast<int>(row_tiles * ksplit);
  int num_sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int grid = n_units < 2 * num_sms ? n_units : 2 * num_sms;  // persistent: two CTAs per SM
  const bool v8 = ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(w.packed)) & 31u) == 0;
  // Programmatic dependent launch: the main loop overlaps the LoRA-down kernel;
  // the epilogue waits for it (griddepcontrol.wait) before reading T.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kDecodeWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const __nv_bfloat16* Xb = reinterpret_cast<const __nv_bfloat16*>(X);
  const __nv_bfloat16* Bb = reinterpret_cast<const __nv_bfloat16*>(B);
  __nv_bfloat16* Yb = reinterpret_cast<__nv_bfloat16*>(Y);
  const int Mi = static_cast<int>(M);
  cudaError_t e;
  if (M <= 8) {
    if (v8)
      e = cudaLaunchKernelEx(&cfg, k_decode<1, true>, w.packed, w.absmax_q, w.dq_scale, w.mean, Xb, Mi, w.N, w.K,
                             static_cast<const float*>(T), Bb, r, s, Yb, partial, counters, ksplit, n_units, cb);
    else
      e = cudaLaunchKernelEx(&cfg, k_decode<1, false>, w.packed, w.absmax_q, w.dq_scale, w.mean, Xb, Mi, w.N, w.K,
                             static_cast<const float*>(T), Bb, r, s, Yb, partial, counters, ksplit, n_units, cb);
  } else {
    if (v8)
      e = cudaLaunchKernelEx(&cfg, k_decode<2, true>, w.packed, w.absmax_q, w.dq_scale, w.mean, Xb, Mi, w.N, w.K,
                             static_cast<const float*>(T), Bb, r, s, Yb, partial, counters, ksplit, n_units, cb);
    else
      e = cudaLaunchKernelEx(&cfg, k_decode<2, false>, w.packed, w.absmax_q, w.dq_scale, w.mean, Xb, Mi, w.N, w.K,
                             static_cast<const float*>(T), Bb, r, s, Yb, partial, counters, ksplit, n_units, cb);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace qlora
