// Decode-shaped QLoRA forward (M <= 16 tokens) with the token values resident
// in shared memory ("QLoRA vs ChatGPT", capability 5: the frozen weight is
// dequantized on the fly, block by block; capability 2: the LoRA term beside
// it).
//
// Y[M, N] = X W'^T + s T B^T, T = X A^T from the LoRA-down kernel that runs
// first (k_lora_t_small in decode.cu).
//
// Used where it measured faster than the TMA-ring kernel of decode.cu (up to 4
// tokens on most weights from 4 M entries, up to 8 on tall ones; the rule is in
// res_plan) and X (M x K bf16, padded) fits in shared memory beside the
// reduction slots.
//
// Work items are (16-row tile, 256-wide K superblock) pairs in tile-major
// order, and every warp of the grid takes one contiguous, equally sized range
// of them, so all warps decode the same number of weights. Since only the
// packed codes stream from memory (X was copied to shared memory once per CTA),
// item ranges need not be shared by the warps of a CTA, and most tiles lie
// within the consecutive warps of one CTA: their pieces are summed through
// shared memory. Only the tiles that straddle two CTAs go through global slots
// and a ticket counter. The last warp of each CTA walks its range backwards, so
// that the pieces of both straddling tiles of a CTA are the first work of the
// warps that hold them.
//
// Within an item the weight is the A operand of mma.sync m16n8k16 (16 rows x 16
// k, bf16 in, fp32 accumulate) and the tokens are its N dimension. Lane (g, t)
// supplies k-slots {2t, 2t+1, 2t+8, 2t+9} of each MMA from the 64 consecutive
// weights of block 4 sb + t of rows g and g + 8 and the matching token values
// (the reduction index is permuted, X alike), so each lane decodes whole
// 64-weight blocks with one 16-entry bf16 table per block, bit-identical to the
// standalone dequant. A lane loads its two blocks' codes (2 x 32 bytes) with
// plain global loads one item ahead (also across tiles), and prefetches the
// item after that into L2.
//
// The LoRA term of a tile, s (T B^T) for its 16 rows, is added to the piece of
// the warp that decodes the tile's last superblock, right after that item, so
// that the warp completing the tile only sums the pieces and stores Y.
//
// Every sum runs in an order fixed by the shapes (pieces in warp order within a
// CTA, then CTAs in order; the LoRA term in one fixed piece), so repeated calls
// give identical bits.
#include "common.cuh"
#include "kernels.h"
#include "lora_tile.cuh"
#include "nf4_lut.cuh"

namespace qlora {
namespace {

constexpr int kResWarps = 16;                 // consumer warps per CTA (one CTA per SM)
constexpr int kXBlockBytes = 64 * 2 + 16;     // one 64-k block of one token, padded for bank spread
// Registers per thread: 16 warps x 112 leave 8192 of the SM's registers free,
// so that a 128-thread CTA of the LoRA-down kernel that precedes this one fits
// beside a CTA of this one. (20 warps x 96 registers with a 64-thread LoRA-down
// CTA measured slower: 24.9 against 19.7 us for 11008x4096 at M = 1, the
// LoRA-down's latency then showing before the tile epilogue.)
constexpr int kResRegs = 112;
// Most dynamic shared memory a CTA of this kernel uses (X copy, slots and
// counters); larger plans go to the TMA-ring kernel. The kernel's limit is set
// to this once, so that every plan up to it launches.
constexpr int kResSmemCap = 200 * 1024;

__device__ __forceinline__ void lookup4(const Nf4Lut& L, uint32_t s, uint32_t sel, uint32_t& o01, uint32_t& o23) {
  const uint32_t lo = prmt(prmt(L.lo[0], L.lo[1], s), prmt(L.lo[2], L.lo[3], s), sel);
  const uint32_t hi = prmt(prmt(L.hi[0], L.hi[1], s), prmt(L.hi[2], L.hi[3], s), sel);
  o01 = prmt(lo, hi, 0x5140);
  o23 = prmt(lo, hi, 0x7362);
}

__device__ __forceinline__ uint4 lds128r(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

__device__ __forceinline__ unsigned int atom_add_acq_rel_cta_shared(uint32_t addr, unsigned int v) {
  unsigned int old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ unsigned int atom_add_acq_rel_gpu_r(unsigned int* p, unsigned int v) {
  unsigned int old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Owner unit of item i when n_items items are cut into n_units ranges
// [u * n_items / n_units, (u + 1) * n_items / n_units).
__host__ __device__ __forceinline__ int64_t owner_of(int64_t i, int64_t n_items, int64_t n_units) {
  return ((i + 1) * n_units - 1) / n_items;
}
__host__ __device__ __forceinline__ int64_t range_begin(int64_t u, int64_t n_items, int64_t n_units) {
  return u * n_items / n_units;
}

struct ResParams {
  const uint8_t* packed;
  const int8_t* q;
  const float* dqs;
  const float* mean;
  const float* absmax;
  const __nv_bfloat16* X;
  const float* T;
  const __nv_bfloat16* Bl;
  __nv_bfloat16* Y;
  float* gpart;            // [n_tiles][max_cta_seg][32 lanes][4 MT] fp32
  unsigned int* gcnt;      // [n_tiles], zeroed by the LoRA-down kernel
  int64_t N, K;
  int64_t n_items, n_units;
  int M, r;
  float s;
  int x_stride;            // bytes per token row of the shared X copy
  int p_max;               // reduction slots per warp
  int cta_tiles;           // CTA-local tile counters per CTA
  int max_cta_seg;         // most CTAs holding pieces of one tile
};

// Shared memory: X [M][x_stride] | slots [kResWarps][p_max][32][4 MT] fp32 | counters [cta_tiles] u32
__host__ __device__ inline size_t res_slot_off(const ResParams& p) {
  return (static_cast<size_t>(p.M) * p.x_stride + 15) / 16 * 16;
}

// A warp has finished its piece of tile `tile`. Store the piece in the warp's
// shared slot; the last of the CTA's warps holding pieces of the tile sums them
// in warp order. A tile that other CTAs hold pieces of too goes on through a
// global slot and ticket; the CTA that brings the last piece sums the CTAs'
// pieces in CTA order. Whoever completes the tile writes Y.
template <int MT>
__device__ __forceinline__ void publish(const float (&acc)[2][MT][4], int64_t tile, int lane, int warp,
                                        float* slots, uint32_t cnt_base, const int64_t* s_wbeg,
                                        const int64_t* s_wtile, const ResParams& p) {
  const int64_t nsb = (p.K / 64 + 3) / 4;
  const int64_t cta = blockIdx.x;
  const int64_t tb = tile * nsb, te = tb + nsb;  // the tile's items
  // this CTA's warps holding pieces of the tile: warp w holds items
  // [s_wbeg[w], s_wbeg[w + 1]), and the holders are consecutive around this warp
  int lw0 = warp, lw1 = warp;
  while (lw0 > 0 && s_wbeg[lw0] > tb) --lw0;
  while (lw1 < kResWarps - 1 && s_wbeg[lw1 + 1] < te) ++lw1;
  const int n_local = lw1 - lw0 + 1;
  constexpr int kSlot = 32 * 4 * MT;  // floats per warp slot
  // this warp's slot for the tile: index = tile - first tile of the warp's range
  float* my_slot = slots + (static_cast<int64_t>(warp) * p.p_max + (tile - s_wtile[warp])) * kSlot;
  float y[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    y[m][0] = acc[0][m][0] + acc[1][m][0];
    y[m][1] = acc[0][m][1] + acc[1][m][1];
    y[m][2] = acc[0][m][2] + acc[1][m][2];
    y[m][3] = acc[0][m][3] + acc[1][m][3];
  }
  if (n_local > 1) {
#pragma unroll
    for (int m = 0; m < MT; ++m)
      reinterpret_cast<float4*>(my_slot + lane * 4 * MT)[m] = make_float4(y[m][0], y[m][1], y[m][2], y[m][3]);
    __syncwarp();  // the lanes' slot stores are ordered before lane 0's release below
    unsigned int old = 0;
    if (lane == 0)
      old = atom_add_acq_rel_cta_shared(cnt_base + static_cast<uint32_t>(tile - s_wtile[0]) * 4u, 1u);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != static_cast<unsigned int>(n_local - 1)) return;  // another warp of the CTA finishes the tile
    __syncwarp();  // lane 0's acquire is ordered before every lane's reads of the slots
#pragma unroll
    for (int m = 0; m < MT; ++m) y[m][0] = y[m][1] = y[m][2] = y[m][3] = 0.0f;
    for (int w = lw0; w <= lw1; ++w) {  // warp order
      const float* sl = slots + (static_cast<int64_t>(w) * p.p_max + (tile - s_wtile[w])) * kSlot;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float4 v = reinterpret_cast<const float4*>(sl + lane * 4 * MT)[m];
        y[m][0] += v.x; y[m][1] += v.y; y[m][2] += v.z; y[m][3] += v.w;
      }
    }
  }
  if (tb < s_wbeg[0] || te > s_wbeg[kResWarps]) {  // pieces in other CTAs too
    // CTAs holding the tile's first and last items (the divisions only on this
    // path: at most two tiles per CTA)
    const int64_t cf = owner_of(tb, p.n_items, p.n_units) / kResWarps;
    const int64_t cl = owner_of(te - 1, p.n_items, p.n_units) / kResWarps;
    float* tp = p.gpart + static_cast<int64_t>(tile) * p.max_cta_seg * kSlot;
#pragma unroll
    for (int m = 0; m < MT; ++m)
      __stcg(reinterpret_cast<float4*>(tp + (cta - cf) * kSlot + lane * 4 * MT) + m,
             make_float4(y[m][0], y[m][1], y[m][2], y[m][3]));
    __syncwarp();
    unsigned int ticket = 0;
    if (lane == 0) ticket = atom_add_acq_rel_gpu_r(&p.gcnt[tile], 1u);
    ticket = __shfl_sync(0xffffffffu, ticket, 0);
    if (ticket != static_cast<unsigned int>(cl - cf)) return;  // another CTA completes the tile
    __syncwarp();
#pragma unroll
    for (int m = 0; m < MT; ++m) y[m][0] = y[m][1] = y[m][2] = y[m][3] = 0.0f;
    for (int64_t c = 0; c <= cl - cf; ++c) {  // CTA order
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(tp + c * kSlot + lane * 4 * MT) + m);
        y[m][0] += v.x; y[m][1] += v.y; y[m][2] += v.z; y[m][3] += v.w;
      }
    }
  }
  store_tile_y<MT>(y, tile, lane, p.Y, p.M, p.N);
}

// SINGLE: single-level storage (the block constant is absmax[b]); V8: the packed
// codes are 32-byte aligned, so each block is one 256-bit load.
template <int MT, bool SINGLE>
__global__ void __maxnreg__(kResRegs)
k_decode_res(const __grid_constant__ ResParams p, const __grid_constant__ Nf4Codebook cb) {
  extern __shared__ __align__(16) uint8_t res_sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t K = p.K, N = p.N;
  const int nkb_row = static_cast<int>(K / 64);
  const int nsb = (nkb_row + 3) / 4;
  const int nblk_pad = nsb * 4;
  const int M = p.M;
  float* slots = reinterpret_cast<float*>(res_sm + res_slot_off(p));
  unsigned int* cnt = reinterpret_cast<unsigned int*>(slots + static_cast<size_t>(kResWarps) * p.p_max * 32 * 4 * MT);
  const uint32_t cnt_base = smem_u32(cnt);

  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kResWarps + warp;
  // this warp's items [i0, i1) (warps numbered n_units and above: none)
  const int64_t i0 = range_begin(gw < p.n_units ? gw : p.n_units, p.n_items, p.n_units);
  const int64_t i1 = range_begin(gw < p.n_units ? gw + 1 : p.n_units, p.n_items, p.n_units);
  const int n_my = static_cast<int>(i1 - i0);
  // the CTA's warp ranges and first tiles, for the tile epilogue
  __shared__ int64_t s_wbeg[kResWarps + 1];
  __shared__ int64_t s_wtile[kResWarps];
  if (lane == 0) {
    s_wbeg[warp] = i0;
    s_wtile[warp] = i0 / nsb;
  }
  if (threadIdx.x == 0) {
    const int64_t u = static_cast<int64_t>(blockIdx.x + 1) * kResWarps;
    s_wbeg[kResWarps] = range_begin(u < p.n_units ? u : p.n_units, p.n_items, p.n_units);
  }
  const bool reverse = warp == kResWarps - 1;
  const int step = reverse ? -1 : 1;
  const int64_t ifirst = reverse ? i1 - 1 : i0;

  // Fetch state, one item ahead of the compute: tile and superblock of the
  // item being loaded and this lane's rows of that tile (rows g and g + 8).
  int64_t ftile = n_my > 0 ? ifirst / nsb : 0;
  int fsb = static_cast<int>(ifirst - ftile * nsb);
  const uint8_t* pa = nullptr;  // packed codes of row g, block t of superblock 0
  const uint8_t* pb = nullptr;
  uint32_t ba0 = 0, bb0 = 0;    // block index of (row, block t of superblock 0)
  bool rowa = false, rowb = false;
  auto set_tile = [&](int64_t tl) {
    const int64_t na = tl * 16 + g, nb = na + 8;
    rowa = na < N;
    rowb = nb < N;
    ba0 = static_cast<uint32_t>(na * nkb_row + t);
    bb0 = static_cast<uint32_t>(nb * nkb_row + t);
    pa = p.packed + static_cast<int64_t>(ba0) * 32;
    pb = p.packed + static_cast<int64_t>(bb0) * 32;
  };
  // Codes and raw block constants of the fetched item. The constants are
  // combined only when the item is decoded, so that no instruction waits on
  // these loads before then. Blocks outside the weight read zero codes and
  // zero constants; their token values in shared memory are zero.
  uint4 ca0, ca1, cb0, cb1;
  int qa = 0, qb = 0;        // int8 codes of the block constants (double-quantized storage)
  float da = 0.0f, db = 0.0f;  // their group scales, or the fp32 constants (single-level)
  auto fetch = [&](int sbk) {
    const bool va = rowa && sbk * 4 + t < nkb_row, vb = rowb && sbk * 4 + t < nkb_row;
    const uint32_t o = static_cast<uint32_t>(sbk) * 128u;  // 4 blocks x 32 bytes
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    ca0 = va ? ldg_stream(pa + o) : z;
    ca1 = va ? ldg_stream(pa + o + 16) : z;
    cb0 = vb ? ldg_stream(pb + o) : z;
    cb1 = vb ? ldg_stream(pb + o + 16) : z;
    const uint32_t ia = ba0 + static_cast<uint32_t>(sbk) * 4u, ib = bb0 + static_cast<uint32_t>(sbk) * 4u;
    if (SINGLE) {
      da = va ? __ldg(p.absmax + ia) : 0.0f;
      db = vb ? __ldg(p.absmax + ib) : 0.0f;
    } else {
      qa = va ? static_cast<int>(__ldg(p.q + ia)) : 0;
      qb = vb ? static_cast<int>(__ldg(p.q + ib)) : 0;
      da = va ? __ldg(p.dqs + (ia >> 8)) : 0.0f;
      db = vb ? __ldg(p.dqs + (ib >> 8)) : 0.0f;
    }
  };
  if (n_my > 0) {  // the first item's loads overlap the X copy below
    set_tile(ftile);
    fetch(fsb);
  }

  // ---- prologue: counters, and X copied into shared memory (padded blocks,
  // zero beyond K). X is an input of the call, complete before the LoRA-down
  // kernel that precedes this one started.
  for (int i = threadIdx.x; i < p.cta_tiles; i += blockDim.x) cnt[i] = 0u;
  {
    const int chunks = M * nblk_pad * 8;  // 16-byte chunks of X to place
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      const int m = c / (nblk_pad * 8);
      const int rem = c - m * nblk_pad * 8;
      const int b = rem >> 3, q = rem & 7;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (b < nkb_row) v = __ldg(reinterpret_cast<const uint4*>(p.X + static_cast<int64_t>(m) * K + b * 64) + q);
      *reinterpret_cast<uint4*>(res_sm + m * p.x_stride + b * kXBlockBytes + q * 16) = v;
    }
  }
  __syncthreads();

  const float mu = SINGLE ? 0.0f : __ldg(p.mean);
  const uint32_t xbase = smem_u32(res_sm);
  // token rows of this lane's B fragments (tokens >= M read the last token:
  // those output columns are never stored)
  uint32_t xrow[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) xrow[m] = xbase + static_cast<uint32_t>(min(g + 8 * m, M - 1) * p.x_stride);

  bool entered = false;  // waited for the LoRA-down kernel (T, zeroed tickets)
  if (n_my > 0) {
    // compute position: tile and superblock of the item being decoded, stepped
    // by +-1 item (no divisions in the loop)
    int64_t tile = ftile;
    int sb = fsb;
    float acc[2][MT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[h][m][0] = acc[h][m][1] = acc[h][m][2] = acc[h][m][3] = 0.0f;
    // L2 prefetch of the tile's LoRA-up rows of B (read by the warp that decodes its last superblock)
    if (lane < 16 && tile * 16 + lane < N) prefetch_l2(p.Bl + (tile * 16 + lane) * p.r);
#pragma unroll 1
    for (int e = 0; e < n_my; ++e) {
      const float mA = SINGLE ? da : __fmaf_rn(static_cast<float>(qa), da, mu);
      const float mB = SINGLE ? db : __fmaf_rn(static_cast<float>(qb), db, mu);
      const Nf4Lut la = make_nf4_lut(cb, mA);
      const Nf4Lut lb = make_nf4_lut(cb, mB);
      const uint4 xa0 = ca0, xa1 = ca1, xb0 = cb0, xb1 = cb1;
      if (e + 1 < n_my) {  // load the next item (in this tile or the neighbouring one)
        fsb += step;
        if (fsb < 0 || fsb >= nsb) {
          ftile += step;
          fsb = reverse ? nsb - 1 : 0;
          set_tile(ftile);
          if (lane < 16 && ftile * 16 + lane < N) prefetch_l2(p.Bl + (ftile * 16 + lane) * p.r);
        }
        fetch(fsb);
        const int sbp = fsb + step;  // and the one after it into L2, when in the same tile
        if (t == 0 && e + 2 < n_my && sbp >= 0 && sbp < nsb) {
          if (rowa) prefetch_l2(pa + static_cast<uint32_t>(sbp) * 128u);
          if (rowb) prefetch_l2(pb + static_cast<uint32_t>(sbp) * 128u);
        }
      }
      const uint32_t xblk = static_cast<uint32_t>((sb * 4 + t) * kXBlockBytes);
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // 16-byte half c of the lane's 32 code bytes: words 4c .. 4c + 3
        const uint4 ca = c ? xa1 : xa0;
        const uint4 cbw = c ? xb1 : xb0;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * c + jj;  // group: k = 16 j .. 16 j + 15 of the block
#pragma unroll
          for (int h = 0; h < 2; ++h) {  // word 2 j + h holds k = 16 j + 8 h .. + 7
            uint4 xv[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) xv[m] = lds128r(xrow[m] + xblk + (16 * j + 8 * h) * 2);
            const uint32_t wa = jj ? (h ? ca.w : ca.z) : (h ? ca.y : ca.x);
            const uint32_t wb = jj ? (h ? cbw.w : cbw.z) : (h ? cbw.y : cbw.x);
            const uint32_t sa = wa & 0x77777777u, sbw = wb & 0x77777777u;
            const uint32_t ta = ((wa >> 1) & 0x44444444u) | 0x32103210u;
            const uint32_t tb = ((wb >> 1) & 0x44444444u) | 0x32103210u;
#pragma unroll
            for (int half = 0; half < 2; ++half) {  // k = 16 j + 8 h + 4 half .. + 3
              uint32_t a0, a1, a2, a3;
              lookup4(la, half ? (sa >> 16) : sa, half ? (ta >> 16) : ta, a0, a2);     // row g
              lookup4(lb, half ? (sbw >> 16) : sbw, half ? (tb >> 16) : tb, a1, a3);   // row g + 8
#pragma unroll
              for (int m = 0; m < MT; ++m)
                mma_bf16_16816(acc[half][m], a0, a1, a2, a3, half ? xv[m].z : xv[m].x, half ? xv[m].w : xv[m].y);
            }
          }
        }
      }
      if (sb == nsb - 1) {  // the tile's last superblock: its LoRA term goes into this piece
        if (!entered) {  // T and the zeroed tickets come from the preceding LoRA-down kernel
          pdl_enter();
          entered = true;
        }
        lora_tile_accumulate<MT>(acc[0], tile, lane, p.T, p.Bl, p.r, p.s, p.M, p.N);
      }
      int sbn = sb + step;
      if (sbn < 0 || sbn >= nsb || e + 1 == n_my) {  // end of this warp's piece of `tile`
        if (!entered) {
          pdl_enter();
          entered = true;
        }
        publish<MT>(acc, tile, lane, warp, slots, cnt_base, s_wbeg, s_wtile, p);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int m = 0; m < MT; ++m) acc[h][m][0] = acc[h][m][1] = acc[h][m][2] = acc[h][m][3] = 0.0f;
        tile += step;
        sbn = reverse ? nsb - 1 : 0;
      }
      sb = sbn;
    }
  }
  // every path waits for the preceding grid before the next one may launch
  if (!entered) pdl_enter();
}

}  // namespace

// Work split and shared-memory plan of the X-resident kernel; ok == false when X
// and the slots do not fit (the TMA-ring kernel then serves the call).
ResPlan res_plan(int64_t M, int64_t N, int64_t K, int num_sms, bool force) {
  ResPlan p{};
  p.ok = false;
  if (M < 1 || M > 16 || N < 1 || K < 64) return p;
  if ((N + 16) * (K / 64) >= (int64_t(1) << 31)) return p;  // block indices are 32-bit in the kernel
  p.mt = M <= 8 ? 1 : 2;
  const int64_t nkb_row = K / 64;
  const int64_t nsb = (nkb_row + 3) / 4;
  p.n_tiles = (N + 15) / 16;
  p.n_items = p.n_tiles * nsb;
  p.grid = num_sms;
  if (p.n_items < static_cast<int64_t>(num_sms) * kResWarps) {
    // fewer items than warps: fewer CTAs, so that no warp is idle
    p.grid = static_cast<int>((p.n_items + kResWarps - 1) / kResWarps);
    if (p.grid < 1) p.grid = 1;
  }
  // at most one warp per item, so that every working warp's range is non-empty
  // and the owners of a tile's items are consecutive working warps (warps
  // numbered n_units and above, in the last CTA, have no range)
  p.n_units = static_cast<int64_t>(p.grid) * kResWarps;
  if (p.n_units > p.n_items) p.n_units = p.n_items;
  // token row stride: whole padded blocks, then rounded to 64 mod 128 bytes so
  // the 8 lanes of each shared-memory phase hit 8 distinct 16-byte bank groups
  int64_t xs = nsb * 4 * kXBlockBytes;
  xs = (xs + 63) / 128 * 128 + 64;
  p.x_stride = static_cast<int>(xs);
  // Reduction slots and counters, from bounds that need no loop over the
  // ranges: a range of L consecutive items touches at most ceil((L - 1) / nsb)
  // + 1 tiles, every warp range holds at most ceil(n_items / n_units) items
  // and every CTA range at most kResWarps times that; a tile's nsb items are
  // held by at most ceil((nsb - 1) / Lc) + 1 CTAs, Lc the fewest items of a
  // CTA range (kResWarps * floor(n_items / n_units), or the last CTA's share).
  const int64_t lw = (p.n_items + p.n_units - 1) / p.n_units;
  const int64_t pmax = (lw - 1 + nsb - 1) / nsb + 1;
  const int64_t lc_max = lw * kResWarps;
  const int64_t ctiles = (lc_max - 1 + nsb - 1) / nsb + 1;
  int64_t lc_min = (p.n_items / p.n_units) * kResWarps;
  const int64_t last_units = p.n_units - static_cast<int64_t>(p.grid - 1) * kResWarps;  // warps of the last CTA
  const int64_t last_min = (p.n_items / p.n_units) * last_units;
  if (last_min < lc_min) lc_min = last_min;
  if (lc_min < 1) lc_min = 1;
  const int64_t maxcs = (nsb - 1 + lc_min - 1) / lc_min + 1;
  p.p_max = static_cast<int>(pmax);
  p.cta_tiles = static_cast<int>(ctiles);
  p.max_cta_seg = static_cast<int>(maxcs);
  const size_t xbytes = (static_cast<size_t>(M) * p.x_stride + 15) / 16 * 16;
  const size_t sbytes = static_cast<size_t>(kResWarps) * p.p_max * 32 * 4 * p.mt * sizeof(float);
  p.smem = xbytes + sbytes + static_cast<size_t>(p.cta_tiles) * 4;
  // Measured crossover against the TMA-ring kernel (B200, L2-cold weights, CUDA
  // graph replay of the whole call, M = 1 / 2 / 4 / 8 tokens): this kernel is
  // faster on square and wide-K-short weights up to 4 tokens (4096x4096: 11.5 /
  // 12.5 / 12.5 against 13.1 / 13.3 / 13.7 us; 2048x2048 from 7.6 against 8.1;
  // 8192x22016 at 1 and 2 tokens: 49.6 / 51.5 against 61.4 / 63.0) and on tall
  // weights (N > K) up to 8 tokens (11008x4096: 17.7 / 18.0 / 18.6 / 19.5
  // against 21.3 / 21.6 / 21.8 / 22.2); it is slower on K > N below 2^26
  // entries (4096x11008: 24.1 / 26.6 / 29.6 against 22.9 / 23.5 / 23.9) and
  // at 8 tokens on square weights (4096x4096: 17.1 against 14.4; 8192x8192 is
  // the exception, 26.6 against 28.5, left to the ring kernel). With two token
  // tiles (9 to 16 tokens) it is slower on every measured shape but the
  // smallest (at 12 / 16 tokens, 11008x4096: 33.6 / 38.2 against 26.0 / 26.8;
  // 4096x4096: 26.6 / 30.5 against 18.4 / 19.1; 2048x2048: 10.9 / 12.2 against
  // 12.3 / 13.1), so it serves at most 8.
  const int64_t nw = N * K;
  const bool faster = (M <= 4 && nw >= (int64_t(1) << 22) && !(K > N && nw < (int64_t(1) << 26))) ||
                      (M <= 8 && K < N && nw >= (int64_t(1) << 24));
  p.ok = (faster || force) && p.smem <= static_cast<size_t>(kResSmemCap);
  return p;
}

size_t res_partial_elems(const ResPlan& p) {
  return static_cast<size_t>(p.n_tiles) * p.max_cta_seg * 32 * 4 * p.mt;
}

cudaError_t launch_decode_res_main(const Nf4View& w, const void* X, int64_t M, const void* B, int r, float s,
                                   void* Y, const float* T, float* partial, unsigned int* counters,
                                   const ResPlan& rp, const float codebook[16], cudaStream_t stream) {
  Nf4Codebook cb;
  for (int i = 0; i < 16; ++i) cb.c[i] = codebook[i];
  ResParams p;
  p.packed = w.packed;
  p.q = w.absmax_q;
  p.dqs = w.dq_scale;
  p.mean = w.mean;
  p.absmax = w.absmax;
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.T = T;
  p.Bl = static_cast<const __nv_bfloat16*>(B);
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.gpart = partial;
  p.gcnt = counters;
  p.N = w.N;
  p.K = w.K;
  p.n_items = rp.n_items;
  p.n_units = rp.n_units;
  p.M = static_cast<int>(M);
  p.r = r;
  p.s = s;
  p.x_stride = rp.x_stride;
  p.p_max = rp.p_max;
  p.cta_tiles = rp.cta_tiles;
  p.max_cta_seg = rp.max_cta_seg;
  const bool single = w.absmax != nullptr;
  const int smem = static_cast<int>(rp.smem);
  cudaError_t e;
  if (rp.mt == 1) {
    if (single) {
      if ((e = ensure_smem_limit<k_decode_res<1, true>>(kResSmemCap)) != cudaSuccess) return e;
      e = launch_pdl(k_decode_res<1, true>, dim3(rp.grid), dim3(kResWarps * 32), smem, stream, p, cb);
    } else {
      if ((e = ensure_smem_limit<k_decode_res<1, false>>(kResSmemCap)) != cudaSuccess) return e;
      e = launch_pdl(k_decode_res<1, false>, dim3(rp.grid), dim3(kResWarps * 32), smem, stream, p, cb);
    }
  } else {
    if (single) {
      if ((e = ensure_smem_limit<k_decode_res<2, true>>(kResSmemCap)) != cudaSuccess) return e;
      e = launch_pdl(k_decode_res<2, true>, dim3(rp.grid), dim3(kResWarps * 32), smem, stream, p, cb);
    } else {
      if ((e = ensure_smem_limit<k_decode_res<2, false>>(kResSmemCap)) != cudaSuccess) return e;
      e = launch_pdl(k_decode_res<2, false>, dim3(rp.grid), dim3(kResWarps * 32), smem, stream, p, cb);
    }
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace qlora
