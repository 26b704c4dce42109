// Decode-shaped QLoRA forward (M <= 16 tokens), bound by the packed 4-bit
// weights ("QLoRA vs ChatGPT", capability 5: the frozen weight is dequantized
// on the fly, block by block).
//
// Y[M, N] = X W'^T + s T B^T with T = X A^T computed first (k_lora_t_small).
//
// Work items are (16-row tile, 256-wide K superblock) pairs in tile-major order.
// Every warp of the grid takes one contiguous, equally sized range of items, so
// all warps do the same amount of decoding whatever N and K are. Within an item
// the weight is the A operand of mma.sync m16n8k16 (16 rows x 16 k, bf16 in,
// fp32 accumulate) and the tokens are its N dimension. The reduction index is
// permuted: lane (g, t) supplies k-slots {2t, 2t+1, 2t+8, 2t+9} of the item's
// 16 MMAs from the 64 consecutive weights of block 4*sb + t of rows g and g+8
// and the matching token values, so each lane decodes whole 64-weight blocks
// with one 16-entry bf16 table per block (bit-identical to the standalone
// dequant) and byte-permute lookups.
//
// A warp's range covers pieces ("segments") of one or more tiles. At the end of
// a segment the warp stores its fp32 partial sums in a slot of the tile; the
// warp that completes a tile (ticket counter, no waiting) sums the tile's slots
// in slot order, adds the LoRA term s (T B^T) with a bf16 hi/lo split of T on
// the tensor cores, and writes Y. The result depends only on the shapes, not on
// timing.
#include "common.cuh"
#include "kernels.h"
#include "nf4_lut.cuh"

namespace qlora {
namespace {

constexpr int kDecodeWarps = 8;
constexpr int kDecodeCtasPerSm = 2;

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// x >> 16 and x >> 1 as high halves of products, so they can issue on the
// multiply-add pipe instead of the integer ALU that the lookups saturate.
__device__ __forceinline__ uint32_t hi16(uint32_t x) { return __umulhi(x, 0x10000u); }
__device__ __forceinline__ uint32_t shr1(uint32_t x) { return __umulhi(x, 0x80000000u); }

// One lane's 64 codes of a row block and the block's double-quant code and scale.
struct RowBlock {
  uint32_t w[8];
  int qv;
  float sc;
};

template <bool V8>
__device__ __forceinline__ void load_row_block(RowBlock& rb, const uint8_t* __restrict__ packed,
                                               const int8_t* __restrict__ q, const float* __restrict__ dqs,
                                               int64_t blk, bool valid) {
  if (valid) {
    const uint4* p = reinterpret_cast<const uint4*>(packed + blk * 32);
    if (V8) {
      ld_global_cs_v8(p, rb.w);
    } else {
      const uint4 a = __ldcs(p), b = __ldcs(p + 1);
      rb.w[0] = a.x; rb.w[1] = a.y; rb.w[2] = a.z; rb.w[3] = a.w;
      rb.w[4] = b.x; rb.w[5] = b.y; rb.w[6] = b.z; rb.w[7] = b.w;
    }
    rb.qv = static_cast<int>(__ldg(q + blk));
    rb.sc = __ldg(dqs + (blk >> 8));
  } else {  // outside the matrix: zero codes (weight 0)
#pragma unroll
    for (int i = 0; i < 8; ++i) rb.w[i] = 0x77777777u;
    rb.qv = 0;
    rb.sc = 0.0f;
  }
}

// 16 tokens' values (k = 16 j .. 16 j + 15 of one block) for one token row.
template <bool V8>
__device__ __forceinline__ void load_x16(uint32_t (&x)[8], const __nv_bfloat16* __restrict__ p, bool valid) {
  if (!valid) {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = 0u;
  } else if (V8) {
    ld_global_nc_v8(p, x);
  } else {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p)), b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

// Byte-permute lookup of four codes with precomputed selectors: `s` holds the
// low three bits of each code (nibbles 0..3), `sel` picks the table half by
// bit 3. Returns the bf16 pairs for codes (0, 1) and (2, 3).
__device__ __forceinline__ void lookup4_sel(const Nf4Lut& L, uint32_t s, uint32_t sel, uint32_t& o01,
                                            uint32_t& o23) {
  const uint32_t lo = prmt(prmt(L.lo[0], L.lo[1], s), prmt(L.lo[2], L.lo[3], s), sel);
  const uint32_t hi = prmt(prmt(L.hi[0], L.hi[1], s), prmt(L.hi[2], L.hi[3], s), sel);
  o01 = prmt(lo, hi, 0x5140);
  o23 = prmt(lo, hi, 0x7362);
}

// Owner warp of item i when n_items items are cut into n_warps ranges
// [w * n_items / n_warps, (w + 1) * n_items / n_warps).
__host__ __device__ __forceinline__ int64_t item_owner(int64_t i, int64_t n_items, int64_t n_warps) {
  return ((i + 1) * n_warps - 1) / n_items;
}

template <int MT, bool V8>
__global__ void __launch_bounds__(kDecodeWarps * 32, kDecodeCtasPerSm)
k_decode(const uint8_t* __restrict__ packed, const int8_t* __restrict__ q, const float* __restrict__ dqs,
         const float* __restrict__ mean, const __nv_bfloat16* __restrict__ X, int M, int64_t N, int64_t K,
         const float* __restrict__ T, const __nv_bfloat16* __restrict__ Bl, int r, float s,
         __nv_bfloat16* __restrict__ Y, float* __restrict__ partial, unsigned int* __restrict__ counters,
         int64_t n_items, int64_t n_warps, int max_seg, const __grid_constant__ Nf4Codebook cb) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kDecodeWarps + warp;
  if (gw >= n_warps) return;
  const int64_t i_begin = gw * n_items / n_warps;
  const int64_t i_end = (gw + 1) * n_items / n_warps;
  if (i_begin >= i_end) return;

  const int64_t nkb_row = K / 64;
  const int64_t nsb = (nkb_row + 3) / 4;
  const float mu = *mean;
  bool entered = false;  // waited for the LoRA-down kernel (T, zeroed counters)

  // item -> (rows, block) of this lane
  auto row_blocks = [&](int64_t item, RowBlock& ra, RowBlock& rb) {
    const int64_t tile = item / nsb;
    const int64_t kb = (item - tile * nsb) * 4 + t;
    const int64_t na = tile * 16 + g, nb = na + 8;
    const bool kv = kb < nkb_row;
    load_row_block<V8>(ra, packed, q, dqs, na * nkb_row + kb, kv && na < N);
    load_row_block<V8>(rb, packed, q, dqs, nb * nkb_row + kb, kv && nb < N);
  };
  // token values of group j (k = 16 j .. 16 j + 15 of the lane's block) of an item
  auto x_group = [&](int64_t item, int j, uint32_t (&x)[MT][8]) {
    const int64_t kb = (item % nsb) * 4 + t;
    const bool kv = kb < nkb_row;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int tok = g + 8 * m;
      load_x16<V8>(x[m], X + static_cast<int64_t>(tok) * K + kb * 64 + 16 * j, kv && tok < M);
    }
  };

  RowBlock nA, nB;
  uint32_t xn[MT][8];
  row_blocks(i_begin, nA, nB);
  x_group(i_begin, 0, xn);

  int64_t i = i_begin;
  while (i < i_end) {
    const int64_t tile = i / nsb;
    const int64_t seg_end = min(i_end, (tile + 1) * nsb);
    float acc[2][MT][4];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[c][m][0] = acc[c][m][1] = acc[c][m][2] = acc[c][m][3] = 0.0f;

    for (; i < seg_end; ++i) {
      const RowBlock cA = nA, cB = nB;
      const bool more = i + 1 < i_end;
      if (more) row_blocks(i + 1, nA, nB);  // next item's codes stream in while this one is decoded
      const Nf4Lut la = make_nf4_lut(cb, __fmaf_rn(static_cast<float>(cA.qv), cA.sc, mu));
      const Nf4Lut lb = make_nf4_lut(cb, __fmaf_rn(static_cast<float>(cB.qv), cB.sc, mu));
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t xc[MT][8];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int e = 0; e < 8; ++e) xc[m][e] = xn[m][e];
        if (j < 3)
          x_group(i, j + 1, xn);
        else if (more)
          x_group(i + 1, 0, xn);
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // word 2j + h holds k = 16 j + 8 h .. + 7
          const uint32_t wa = cA.w[2 * j + h], wb = cB.w[2 * j + h];
          const uint32_t sa = wa & 0x77777777u, sb = wb & 0x77777777u;
          const uint32_t ta = (shr1(wa) & 0x44444444u) | 0x32103210u;
          const uint32_t tb = (shr1(wb) & 0x44444444u) | 0x32103210u;
#pragma unroll
          for (int half = 0; half < 2; ++half) {  // step st = 2 h + half: k = 16 j + 4 st .. + 3
            const int st = 2 * h + half;
            uint32_t a0, a1, a2, a3;
            lookup4_sel(la, half ? hi16(sa) : sa, half ? hi16(ta) : ta, a0, a2);  // row g
            lookup4_sel(lb, half ? hi16(sb) : sb, half ? hi16(tb) : tb, a1, a3);  // row g + 8
#pragma unroll
            for (int m = 0; m < MT; ++m) mma16816(acc[st & 1][m], a0, a1, a2, a3, xc[m][2 * st], xc[m][2 * st + 1]);
          }
        }
      }
    }

    // ---- segment done: publish the partial sums of this tile piece ----
    if (!entered) {  // T and the zeroed counters come from the preceding LoRA-down kernel
      pdl_enter();
      entered = true;
    }
    const int64_t w_first = item_owner(tile * nsb, n_items, n_warps);
    const int64_t w_last = item_owner((tile + 1) * nsb - 1, n_items, n_warps);
    const int nseg = static_cast<int>(w_last - w_first + 1);
    const int slot = static_cast<int>(gw - w_first);
    float* tile_part = partial + static_cast<int64_t>(tile) * max_seg * (32 * 4 * MT);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float4 v = make_float4(acc[0][m][0] + acc[1][m][0], acc[0][m][1] + acc[1][m][1],
                                   acc[0][m][2] + acc[1][m][2], acc[0][m][3] + acc[1][m][3]);
      __stcg(reinterpret_cast<float4*>(tile_part + (slot * 32 + lane) * 4 * MT) + m, v);
    }
    __threadfence();
    __syncwarp();
    unsigned int ticket = 0;
    if (nseg > 1) {
      if (lane == 0) ticket = atomicAdd(&counters[tile], 1u);
      ticket = __shfl_sync(0xffffffffu, ticket, 0);
      if (ticket != static_cast<unsigned int>(nseg - 1)) continue;  // another warp completes the tile
      __threadfence();
    }

    // ---- complete the tile: sum the slots in order, add s (T B^T), store Y ----
    float y[MT][4];
#pragma unroll
    for (int m = 0; m < MT; ++m) y[m][0] = y[m][1] = y[m][2] = y[m][3] = 0.0f;
    for (int sl = 0; sl < nseg; ++sl) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(tile_part + (sl * 32 + lane) * 4 * MT) + m);
        y[m][0] += v.x; y[m][1] += v.y; y[m][2] += v.z; y[m][3] += v.w;
      }
    }
    // LoRA up: rows of B are the A operand, T^T (split into bf16 hi + lo) the B operand.
    const int64_t na = tile * 16 + g, nb = na + 8;
    float l[MT][4];
#pragma unroll
    for (int m = 0; m < MT; ++m) l[m][0] = l[m][1] = l[m][2] = l[m][3] = 0.0f;
    for (int j0 = 0; j0 < r; j0 += 16) {
      const uint32_t b_a0 = na < N ? *reinterpret_cast<const uint32_t*>(Bl + na * r + j0 + 2 * t) : 0u;
      const uint32_t b_a2 = na < N ? *reinterpret_cast<const uint32_t*>(Bl + na * r + j0 + 2 * t + 8) : 0u;
      const uint32_t b_a1 = nb < N ? *reinterpret_cast<const uint32_t*>(Bl + nb * r + j0 + 2 * t) : 0u;
      const uint32_t b_a3 = nb < N ? *reinterpret_cast<const uint32_t*>(Bl + nb * r + j0 + 2 * t + 8) : 0u;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int tok = g + 8 * m;
        float tv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (tok < M) {
          const float* tp = T + static_cast<int64_t>(tok) * r + j0 + 2 * t;
          tv[0] = __ldcg(tp);
          tv[1] = __ldcg(tp + 1);
          tv[2] = __ldcg(tp + 8);
          tv[3] = __ldcg(tp + 9);
        }
        uint32_t hi[2], lo[2];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const uint32_t h = pack_bf16x2(tv[2 * p], tv[2 * p + 1]);
          hi[p] = h;
          lo[p] = pack_bf16x2(tv[2 * p] - bf16lo_to_f32(h), tv[2 * p + 1] - bf16hi_to_f32(h));
        }
        mma16816(l[m], b_a0, b_a1, b_a2, b_a3, hi[0], hi[1]);
        mma16816(l[m], b_a0, b_a1, b_a2, b_a3, lo[0], lo[1]);
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int tok0 = 8 * m + 2 * t, tok1 = tok0 + 1;
      if (na < N) {
        if (tok0 < M) Y[static_cast<int64_t>(tok0) * N + na] = __float2bfloat16_rn(fmaf(s, l[m][0], y[m][0]));
        if (tok1 < M) Y[static_cast<int64_t>(tok1) * N + na] = __float2bfloat16_rn(fmaf(s, l[m][1], y[m][1]));
      }
      if (nb < N) {
        if (tok0 < M) Y[static_cast<int64_t>(tok0) * N + nb] = __float2bfloat16_rn(fmaf(s, l[m][2], y[m][2]));
        if (tok1 < M) Y[static_cast<int64_t>(tok1) * N + nb] = __float2bfloat16_rn(fmaf(s, l[m][3], y[m][3]));
      }
    }
    if (nseg > 1 && lane == 0) counters[tile] = 0u;  // ready for the next call
  }
}

// T[m, j] = sum_k X[m, k] A[j, k] for M <= 16 (fp32 on CUDA cores), one CTA per
// adapter row j, 16-byte loads (8 k per thread and step). Block 0 also clears
// the decode kernel's ticket counters.
template <int MT>
__global__ void __launch_bounds__(256)
k_lora_t_small(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ A, int M, int64_t K, int r,
               float* __restrict__ T, unsigned int* __restrict__ counters, int64_t n_counters) {
  __shared__ float red[8][8 * MT];
  pdl_enter();  // after this, the decode kernel may start its main loop
  const int j = blockIdx.x;
  if (j == 0)
    for (int64_t i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0u;
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

DecodePlan decode_plan(int64_t M, int64_t N, int64_t K, int ref_sms) {
  DecodePlan p;
  p.mt = M <= 8 ? 1 : 2;
  p.row_tiles = (N + 15) / 16;
  p.nsb = (K / 64 + 3) / 4;
  p.n_items = p.row_tiles * p.nsb;
  // At most one warp per item, so every warp's range is non-empty and the
  // owners of consecutive items are consecutive warps (slot = warp - first owner).
  const int64_t cap = static_cast<int64_t>(ref_sms) * kDecodeCtasPerSm * kDecodeWarps;
  p.n_warps = p.n_items < cap ? p.n_items : cap;
  if (p.n_warps < 1) p.n_warps = 1;
  p.grid = static_cast<int>((p.n_warps + kDecodeWarps - 1) / kDecodeWarps);
  p.max_seg = 1;
  for (int64_t tile = 0; tile < p.row_tiles; ++tile) {
    const int64_t a = item_owner(tile * p.nsb, p.n_items, p.n_warps);
    const int64_t b = item_owner((tile + 1) * p.nsb - 1, p.n_items, p.n_warps);
    if (b - a + 1 > p.max_seg) p.max_seg = static_cast<int>(b - a + 1);
  }
  return p;
}

size_t decode_partial_elems(const DecodePlan& p) {
  return static_cast<size_t>(p.row_tiles) * p.max_seg * 32 * 4 * p.mt;
}

size_t decode_counter_words(const DecodePlan& p) { return static_cast<size_t>(p.row_tiles); }

cudaError_t launch_decode_fwd(const Nf4View& w, const void* X, int64_t M, const void* A, const void* B, int r,
                              float s, void* Y, float* T, float* partial, unsigned int* counters,
                              const DecodePlan& p, const float codebook[16], cudaStream_t stream) {
  Nf4Codebook cb;
  for (int i = 0; i < 16; ++i) cb.c[i] = codebook[i];
  const __nv_bfloat16* Xb = reinterpret_cast<const __nv_bfloat16*>(X);
  cudaError_t e = launch_pdl(p.mt == 1 ? k_lora_t_small<1> : k_lora_t_small<2>, dim3(r), dim3(256), 0, stream, Xb,
                             reinterpret_cast<const __nv_bfloat16*>(A), static_cast<int>(M), w.K, r, T, counters,
                             p.row_tiles);
  if (e != cudaSuccess) return e;
  // Programmatic dependent launch: the main loop overlaps the LoRA-down kernel;
  // each warp waits for it (griddepcontrol.wait) before its first ticket.
  const bool v8 = ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(w.packed)) & 31u) == 0;
  const __nv_bfloat16* Bb = reinterpret_cast<const __nv_bfloat16*>(B);
  __nv_bfloat16* Yb = reinterpret_cast<__nv_bfloat16*>(Y);
  const int Mi = static_cast<int>(M);
  auto kern = p.mt == 1 ? (v8 ? k_decode<1, true> : k_decode<1, false>)
                        : (v8 ? k_decode<2, true> : k_decode<2, false>);
  e = launch_pdl(kern, dim3(p.grid), dim3(kDecodeWarps * 32), 0, stream, w.packed, w.absmax_q, w.dq_scale, w.mean,
                 Xb, Mi, w.N, w.K, static_cast<const float*>(T), Bb, r, s, Yb, partial, counters, p.n_items,
                 p.n_warps, p.max_seg, cb);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace qlora
