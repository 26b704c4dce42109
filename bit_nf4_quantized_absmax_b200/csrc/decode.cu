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
// in slot order and writes Y. The LoRA term s (T B^T), with a bf16 hi/lo split
// of T on the tensor cores, goes into the piece of the warp that decodes the
// tile's last superblock. The result depends only on the shapes, not on timing.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "lora_tile.cuh"
#include "nf4_lut.cuh"
#include "tensor_map.h"

namespace qlora {
namespace {

constexpr int kDecodeWarps = 8;

// (Writing these shifts as high halves of products, to move them off the
// integer ALU, measured 4% slower than plain shifts.)
__device__ __forceinline__ uint32_t hi16(uint32_t x) { return x >> 16; }
__device__ __forceinline__ uint32_t shr1(uint32_t x) { return x >> 1; }

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

// Orders this thread's generic-proxy reads of shared memory before later
// async-proxy writes (TMA) to it. The consumer warps read the TMA-filled stages
// with ordinary loads, so each executes it before releasing a stage for the
// next copy; without it, a copy into a released stage was seen to overwrite
// token values that a warp had not read yet.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Owner unit of item i when n_items items are cut into n_units ranges
// [u * n_items / n_units, (u + 1) * n_items / n_units).
__host__ __device__ __forceinline__ int64_t item_owner(int64_t i, int64_t n_items, int64_t n_units) {
  return ((i + 1) * n_units - 1) / n_items;
}

// Ticket of a split tile: release this warp's partial sums, acquire the others'.
__device__ __forceinline__ unsigned int atom_add_acq_rel_gpu(unsigned int* p, unsigned int v) {
  unsigned int old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// End of a work unit's piece of 16-row tile `tile` (item row `item_row` of the
// unit ranges; this unit holds items [i_begin, i_end)): store the warp's fp32
// partial sums in the tile's slot; the warp that brings the tile's last piece
// (ticket counter, no waiting) sums the slots in slot order and writes Y. (The
// tile's LoRA term is already in the piece of the unit that decoded the tile's
// last superblock.)
template <int MT>
__device__ __forceinline__ void publish_segment(const float (&acc)[2][MT][4], int64_t item_row, int64_t tile,
                                                int64_t unit, int lane, int64_t nsb, int64_t i_begin, int64_t i_end,
                                                int64_t n_items, int64_t n_units, int max_seg,
                                                float* __restrict__ partial, unsigned int* __restrict__ counters,
                                                __nv_bfloat16* __restrict__ Y, int M, int64_t N) {
  // units holding the row's first and last items (a division only when the
  // row reaches beyond this unit's range)
  const int64_t gb = item_row * nsb, ge = gb + nsb;
  const int64_t w_first = gb < i_begin ? floor_div_small((gb + 1) * n_units - 1, n_items) : unit;
  const int64_t w_last = ge > i_end ? floor_div_small(ge * n_units - 1, n_items) : unit;
  const int nseg = static_cast<int>(w_last - w_first + 1);
  const int slot = static_cast<int>(unit - w_first);
  float* tile_part = partial + static_cast<int64_t>(tile) * max_seg * (32 * 4 * MT);
  float y[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    y[m][0] = acc[0][m][0] + acc[1][m][0];
    y[m][1] = acc[0][m][1] + acc[1][m][1];
    y[m][2] = acc[0][m][2] + acc[1][m][2];
    y[m][3] = acc[0][m][3] + acc[1][m][3];
  }
  if (nseg > 1) {
#pragma unroll
    for (int m = 0; m < MT; ++m)
      __stcg(reinterpret_cast<float4*>(tile_part + (slot * 32 + lane) * 4 * MT) + m,
             make_float4(y[m][0], y[m][1], y[m][2], y[m][3]));
    __syncwarp();  // the lanes' partial stores are ordered before lane 0's release below
    unsigned int ticket = 0;
    if (lane == 0) ticket = atom_add_acq_rel_gpu(&counters[tile], 1u);
    ticket = __shfl_sync(0xffffffffu, ticket, 0);
    if (ticket != static_cast<unsigned int>(nseg - 1)) return;  // another warp completes the tile
    __syncwarp();  // lane 0's acquire is ordered before every lane's reads of the slots
#pragma unroll
    for (int m = 0; m < MT; ++m) y[m][0] = y[m][1] = y[m][2] = y[m][3] = 0.0f;
    for (int sl = 0; sl < nseg; ++sl) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(tile_part + (sl * 32 + lane) * 4 * MT) + m);
        y[m][0] += v.x; y[m][1] += v.y; y[m][2] += v.z; y[m][3] += v.w;
      }
    }
  }
  store_tile_y<MT>(y, tile, lane, Y, M, N);
}

// CTA items are (128-row group, 256-wide K superblock) pairs in group-major
// order; each CTA takes one contiguous, equally sized range of items. Warp w of
// the 8 consumer warps decodes rows 16 w .. 16 w + 15 of the group. A ninth warp
// feeds a kStages-deep ring by TMA: per stage one box of the packed weights
// (128 rows x 128 bytes) and four boxes of the token values (64 k x 8 MT rows,
// one per 64-weight block of the superblock), all with the 128-byte swizzle so
// that the lanes' 16-byte reads are free of bank conflicts.
constexpr int kStages = 4;
constexpr int kRowsPerItem = kDecodeWarps * 16;
constexpr int kWBytes = kRowsPerItem * 128;

__host__ __device__ constexpr int decode_x_bytes(int mt) { return 4 * 8 * mt * 128; }
__host__ __device__ constexpr int decode_stage_bytes(int mt) { return kWBytes + decode_x_bytes(mt); }
__host__ __device__ constexpr int decode_smem_bytes(int mt) { return kStages * decode_stage_bytes(mt) + 1024; }
constexpr int kDecodeCtasPerSm = 2;

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// SINGLE: single-level storage, the block constant is absmax[b] itself (q, dqs
// and mean unused); otherwise m'_b = fmaf(q[b], dqs[b / 256], mean).
template <int MT, bool SINGLE>
__global__ void __launch_bounds__((kDecodeWarps + 1) * 32, kDecodeCtasPerSm)
k_decode(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
         const int8_t* __restrict__ q, const float* __restrict__ dqs, const float* __restrict__ mean,
         const float* __restrict__ absmax, int M,
         int64_t N, int64_t K, const float* __restrict__ T, const __nv_bfloat16* __restrict__ Bl, int r, float s,
         __nv_bfloat16* __restrict__ Y, float* __restrict__ partial, unsigned int* __restrict__ counters,
         int64_t n_items, int64_t n_ctas, int max_seg, int32_t* __restrict__ err,
         const __grid_constant__ Nf4Codebook cb) {
  constexpr int kStage = decode_stage_bytes(MT);
  extern __shared__ uint8_t dsm_raw[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t empty[kStages];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t cta = blockIdx.x;
  const int64_t i_begin = cta * n_items / n_ctas;
  const int64_t i_end = (cta + 1) * n_items / n_ctas;
  const int n_my = static_cast<int>(i_end - i_begin);
  const int nkb_row = static_cast<int>(K / 64);
  const int nsb = (nkb_row + 3) / 4;
  const int64_t rg0 = i_begin / nsb;  // (row group, superblock) of the first item
  const int sb0 = static_cast<int>(i_begin - rg0 * nsb);
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));

  if (threadIdx.x == 0) {
#pragma unroll
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kDecodeWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (n_my <= 0) return;

  if (warp == kDecodeWarps) {  // ---- producer warp: TMA ring ----
    if (lane == 0) {
      prefetch_tmap(&tm_w);
      prefetch_tmap(&tm_x);
      int64_t rg = rg0;
      int sb = sb0, st = 0;
      uint32_t ph = 0;
      for (int n = 0; n < n_my; ++n) {
        if (n >= kStages && !mbar_wait_bounded(&empty[st], ph ^ 1u, err, DEV_TIMEOUT_SMEM_EMPTY)) break;
        uint8_t* dst = dsm + st * kStage;
        mbar_arrive_expect_tx(&full[st], kStage);
        tma_load_2d(dst, &tm_w, &full[st], sb * 128, static_cast<int32_t>(rg * kRowsPerItem));
#pragma unroll
        for (int b = 0; b < 4; ++b)
          tma_load_2d(dst + kWBytes + b * (8 * MT * 128), &tm_x, &full[st], sb * 256 + 64 * b, 0);
        if (++st == kStages) {
          st = 0;
          ph ^= 1u;
        }
        if (++sb == nsb) {
          sb = 0;
          ++rg;
        }
      }
    }
    // no launch_dependents here: the consumer warps signal the next grid after
    // they have waited for the LoRA-down kernel (wait, then trigger, as in
    // every kernel of the library), so at most two grids are ever in flight
    return;
  }
  // ---- consumer warps ----
  const int g = lane >> 2, t = lane & 3;
  const uint32_t smem0 = smem_u32(dsm);
  // the lane's weight chunks (2t + c) of rows 16 w + g and 16 w + g + 8, and the
  // token rows g + 8 m of its block's token box, under the 128-byte swizzle
  const uint32_t offW0 = (warp * 16 + g) * 128 + (((2 * t) ^ g) << 4);
  const uint32_t offW1 = (warp * 16 + g) * 128 + (((2 * t + 1) ^ g) << 4);
  const uint32_t offX = kWBytes + t * (8 * MT * 128) + g * 128;

  const float mu = SINGLE ? 0.0f : *mean;
  // block constants of rows 16 w + g and + 8 (m' = 0 outside the matrix)
  auto consts = [&](int64_t rg, int sb, int& qa, float& sa, int& qb, float& sbv, bool& va, bool& vb) {
    const int kb = sb * 4 + t;
    const int64_t na = rg * kRowsPerItem + warp * 16 + g, nb = na + 8;
    va = kb < nkb_row && na < N;
    vb = kb < nkb_row && nb < N;
    const int64_t ba = na * nkb_row + kb, bb = nb * nkb_row + kb;
    if (SINGLE) {
      qa = qb = 0;
      sa = va ? __ldg(absmax + ba) : 0.0f;
      sbv = vb ? __ldg(absmax + bb) : 0.0f;
    } else {
      qa = va ? static_cast<int>(__ldg(q + ba)) : 0;
      sa = va ? __ldg(dqs + (ba >> 8)) : 0.0f;
      qb = vb ? static_cast<int>(__ldg(q + bb)) : 0;
      sbv = vb ? __ldg(dqs + (bb >> 8)) : 0.0f;
    }
  };

  int nqa, nqb;
  float nsa, nsc;
  bool nva, nvb;
  consts(rg0, sb0, nqa, nsa, nqb, nsc, nva, nvb);

  bool entered = false;  // waited for the LoRA-down kernel (T, zeroed counters)
  bool ok = true;
  int n = 0, stage = 0;
  uint32_t phase = 0;
  int64_t rg = rg0;
  int sb = sb0;
  while (n < n_my) {
    const int seg_items = min(n_my - n, nsb - sb);  // items of this row group in the CTA's range
    float acc[2][MT][4];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[c][m][0] = acc[c][m][1] = acc[c][m][2] = acc[c][m][3] = 0.0f;

    for (int e = 0; e < seg_items; ++e, ++n, ++sb) {
      const float mA = nva ? (SINGLE ? nsa : __fmaf_rn(static_cast<float>(nqa), nsa, mu)) : 0.0f;
      const float mB = nvb ? (SINGLE ? nsc : __fmaf_rn(static_cast<float>(nqb), nsc, mu)) : 0.0f;
      if (n + 1 < n_my) {  // next item's constants
        const bool wrap = sb + 1 == nsb;
        consts(wrap ? rg + 1 : rg, wrap ? 0 : sb + 1, nqa, nsa, nqb, nsc, nva, nvb);
      }
      const Nf4Lut la = make_nf4_lut(cb, mA);
      const Nf4Lut lb = make_nf4_lut(cb, mB);
      const bool got = mbar_wait_bounded(&full[stage], phase, err, DEV_TIMEOUT_TMA_FULL);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      const uint32_t st = smem0 + static_cast<uint32_t>(stage) * kStage;
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // weight chunk c: words 4c .. 4c + 3 of the lane's block
        const uint4 ca = lds128(st + (c ? offW1 : offW0));
        const uint4 cbk = lds128(st + 8 * 128 + (c ? offW1 : offW0));
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * c + jj;  // group: k = 16 j .. 16 j + 15 of the block
#pragma unroll
          for (int h = 0; h < 2; ++h) {  // word 2j + h holds k = 16 j + 8 h .. + 7
            uint4 xv[MT];  // token values of k = 16 j + 8 h .. + 7: 16-byte chunk 2j + h of the box row
#pragma unroll
            for (int m = 0; m < MT; ++m)
              xv[m] = lds128(st + offX + m * (8 * 128) + (((2 * j + h) ^ g) << 4));
            const uint32_t wa = jj ? (h ? ca.w : ca.z) : (h ? ca.y : ca.x);
            const uint32_t wb = jj ? (h ? cbk.w : cbk.z) : (h ? cbk.y : cbk.x);
            const uint32_t sa = wa & 0x77777777u, sbw = wb & 0x77777777u;
            const uint32_t ta = (shr1(wa) & 0x44444444u) | 0x32103210u;
            const uint32_t tb = (shr1(wb) & 0x44444444u) | 0x32103210u;
#pragma unroll
            for (int half = 0; half < 2; ++half) {  // step 2 h + half: k = 16 j + 8 h + 4 half .. + 3
              uint32_t a0, a1, a2, a3;
              lookup4_sel(la, half ? hi16(sa) : sa, half ? hi16(ta) : ta, a0, a2);    // row g
              lookup4_sel(lb, half ? hi16(sbw) : sbw, half ? hi16(tb) : tb, a1, a3);  // row g + 8
#pragma unroll
              for (int m = 0; m < MT; ++m)
                mma_bf16_16816(acc[half][m], a0, a1, a2, a3, half ? xv[m].z : xv[m].x, half ? xv[m].w : xv[m].y);
            }
          }
        }
      }
      fence_proxy_async_shared();  // this warp's reads of the stage precede the next TMA into it
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);  // this warp is done with the stage
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
      if (sb == nsb - 1) {  // the row's last superblock: the tile's LoRA term goes into this piece
        if (!entered) {  // T and the zeroed counters come from the preceding LoRA-down kernel
          pdl_enter();
          entered = true;
        }
        lora_tile_accumulate<MT>(acc[0], rg * kDecodeWarps + warp, lane, T, Bl, r, s, M, N);
      }
    }
    if (!ok) break;
    if (!entered) {  // T and the zeroed counters come from the preceding LoRA-down kernel
      pdl_enter();
      entered = true;
    }
    publish_segment<MT>(acc, rg, rg * kDecodeWarps + warp, cta, lane, nsb, i_begin, i_end, n_items, n_ctas, max_seg,
                        partial, counters, Y, M, N);
    ++rg;
    sb = 0;
  }
  // a warp that published nothing (a bounded wait gave up) still waits for the
  // LoRA-down kernel before it lets the next grid launch, like every other path
  if (!entered) pdl_enter();
}

// T[m, j] = sum_k X[m, k] A[j, k] for M <= 16 (fp32 on CUDA cores), one CTA per
// adapter row j, 16-byte loads (8 k per thread and step). Block 0 also clears
// the decode kernel's ticket counters. NT threads: 256 before the TMA-ring
// decode kernel; 128 with at most 64 registers before the X-resident one, so
// that one CTA of it fits on an SM beside a CTA of that kernel.
template <int MT, int NT>
__global__ void __launch_bounds__(NT, NT < 256 ? 16 * 64 / NT : 1)
k_lora_t_small(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ A, int M, int64_t K, int r,
               float* __restrict__ T, unsigned int* __restrict__ counters, int64_t n_counters,
               const float* __restrict__ col_scale) {
  constexpr int kLoraDownThreads = NT;
  __shared__ float red[kLoraDownThreads / 32][8 * MT];
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
    for (int w = 0; w < kLoraDownThreads / 32; ++w) v += red[w][threadIdx.x];
    // several adapters at once: each rank column carries its adapter's scale
    if (col_scale) v = __fmul_rn(col_scale[j], v);
    T[static_cast<int64_t>(threadIdx.x) * r + j] = v;
  }
}

}  // namespace

DecodePlan decode_plan(int64_t M, int64_t N, int64_t K, int ref_sms) {
  DecodePlan p;
  p.mt = M <= 8 ? 1 : 2;
  p.n_groups = (N + kRowsPerItem - 1) / kRowsPerItem;
  p.row_tiles = p.n_groups * kDecodeWarps;
  p.nsb = (K / 64 + 3) / 4;
  p.n_items = p.n_groups * p.nsb;
  // At most one CTA per item, so every CTA's range is non-empty and the owners
  // of consecutive items are consecutive CTAs (slot = CTA - first owner).
  const int64_t cap = static_cast<int64_t>(ref_sms) * kDecodeCtasPerSm;
  int64_t grid = p.n_items < cap ? p.n_items : cap;
  if (grid < 1) grid = 1;
  p.grid = static_cast<int>(grid);
  p.max_seg = 1;
  for (int64_t rg = 0; rg < p.n_groups; ++rg) {
    const int64_t a = item_owner(rg * p.nsb, p.n_items, grid);
    const int64_t b = item_owner((rg + 1) * p.nsb - 1, p.n_items, grid);
    if (b - a + 1 > p.max_seg) p.max_seg = static_cast<int>(b - a + 1);
  }
  return p;
}

size_t decode_partial_elems(const DecodePlan& p) {
  return static_cast<size_t>(p.row_tiles) * p.max_seg * 32 * 4 * p.mt;
}

size_t decode_counter_words(const DecodePlan& p) { return static_cast<size_t>(p.row_tiles); }

namespace {

bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  PFN_encodeTiled enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_decode_fwd(const Nf4View& w, const void* X, int64_t M, const void* A, const void* B, int r,
                              float s, void* Y, float* T, float* partial, unsigned int* counters,
                              const DecodePlan& p, const ResPlan& rp, const float codebook[16], int32_t* err,
                              cudaStream_t stream, const float* col_scale) {
  if (rp.ok) {  // token values resident in shared memory (decode_res.cu)
    cudaError_t e = launch_pdl(rp.mt == 1 ? k_lora_t_small<1, 128> : k_lora_t_small<2, 128>, dim3(r), dim3(128), 0, stream,
                               reinterpret_cast<const __nv_bfloat16*>(X), reinterpret_cast<const __nv_bfloat16*>(A),
                               static_cast<int>(M), w.K, r, T, counters, rp.n_tiles, col_scale);
    if (e != cudaSuccess) return e;
    return launch_decode_res_main(w, X, M, B, r, s, Y, T, partial, counters, rp, codebook, stream);
  }
  if (w.N >= (int64_t(1) << 31) || w.K >= (int64_t(1) << 31)) return cudaErrorInvalidValue;  // TMA coordinates
  Nf4Codebook cb;
  for (int i = 0; i < 16; ++i) cb.c[i] = codebook[i];
  // packed weights as a [N, K/2] byte matrix, box = 128 rows x 128 bytes;
  // token values [M, K] bf16, box = 64 k x 8 MT rows (rows >= M read as zero)
  CUtensorMap tw, tx;
  if (!encode_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.packed, static_cast<uint64_t>(w.K / 2),
                 static_cast<uint64_t>(w.N), static_cast<uint64_t>(w.K / 2), 128u, kRowsPerItem) ||
      !encode_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(w.K), static_cast<uint64_t>(M),
                 static_cast<uint64_t>(w.K) * 2, 64u, 8u * p.mt))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(p.mt == 1 ? k_lora_t_small<1, 256> : k_lora_t_small<2, 256>, dim3(r), dim3(256), 0, stream,
                             reinterpret_cast<const __nv_bfloat16*>(X), reinterpret_cast<const __nv_bfloat16*>(A),
                             static_cast<int>(M), w.K, r, T, counters, p.row_tiles, col_scale);
  if (e != cudaSuccess) return e;
  // Programmatic dependent launch: the main loop overlaps the LoRA-down kernel;
  // each consumer warp waits for it (griddepcontrol.wait) before its first ticket.
  const __nv_bfloat16* Bb = reinterpret_cast<const __nv_bfloat16*>(B);
  __nv_bfloat16* Yb = reinterpret_cast<__nv_bfloat16*>(Y);
  const int Mi = static_cast<int>(M);
  const bool single = w.absmax != nullptr;
  auto kern = p.mt == 1 ? (single ? k_decode<1, true> : k_decode<1, false>)
                        : (single ? k_decode<2, true> : k_decode<2, false>);
  const int smem = decode_smem_bytes(p.mt);
  e = p.mt == 1 ? (single ? ensure_smem_limit<k_decode<1, true>>(smem) : ensure_smem_limit<k_decode<1, false>>(smem))
                : (single ? ensure_smem_limit<k_decode<2, true>>(smem) : ensure_smem_limit<k_decode<2, false>>(smem));
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(p.grid), dim3((kDecodeWarps + 1) * 32), smem, stream, tw, tx, w.absmax_q, w.dq_scale,
                 w.mean, w.absmax, Mi, w.N, w.K, static_cast<const float*>(T), Bb, r, s, Yb, partial, counters,
                 p.n_items, static_cast<int64_t>(p.grid), p.max_seg, err, cb);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace qlora
