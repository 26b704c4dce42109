// Persistent tcgen05 GEMM for sm_100a: TMA loads into 128-byte-swizzled shared
// memory, one thread issues tcgen05.mma (bf16 x bf16 -> fp32) into a
// double-buffered TMEM accumulator, four epilogue warps drain TMEM with
// tcgen05.ld while the next tile's mainloop runs.
//
//   C[M, Nc] = A1[M, K1] op(B1) + A2[M, K2] op(B2)
//
// The second pair ("slab") carries the rank-r LoRA term: for the forward pass
// [X | s T] [W' | B]^T, for dX [dY | s U] [W' ; A] ("QLoRA vs ChatGPT",
// capability 2: the adapter sits beside the frozen weight; capability 5: it is
// the only part that receives gradients). A and B may each be K-major (the
// reduction index contiguous) or MN-major (the output index contiguous); the
// TMA boxes and UMMA shared-memory descriptors follow the operand's layout.
//
// Warp roles (192 threads): warp 0 issues TMA, warp 1 allocates TMEM and issues
// MMAs, warps 2..5 run the epilogue (warp w reads TMEM lanes 32*(w%4)..+31).
// Every mbarrier wait is bounded; a timeout records an error word and makes the
// CTA leave its loops.
#include <cuda.h>

#include <atomic>
#include <cstdlib>
#include <random>

#include "common.cuh"
#include "kernels.h"
#include "nf4_lut.cuh"
#include "tensor_map.h"

namespace qlora {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;

enum OutMode : int { OUT_BF16 = 0, OUT_LORA = 1, OUT_PARTIAL = 2 };

struct EpiParams {
  void* C; int64_t ldc;                    // OUT_BF16: bf16 [M, ldc]
  float* f32; int64_t ld_f32;              // OUT_LORA: optional fp32 copy [M, ld_f32] (cols < Nc)
  void* s_bf16; void* hi; void* lo;        // OUT_LORA: bf16 [M, ld_pad]: s*C, C, C - bf16(C)
  int64_t ld_pad; float s;
  float* P;                                // OUT_PARTIAL: fp32 [splits][M][Nc]
};

struct TileSched {
  int tiles_m, tiles_n, splits;
  int nkb;        // total k-blocks (main + slab)
  int nk1;        // k-blocks of the main pair
  int kb_per_split;
  int group_m;    // 0: tiles M-fastest; else (one split) bands of group_m M tiles, M-fastest inside a band
  // 2-CTA kernels: units [0, full_units) are whole tiles; the remaining tail_tiles
  // tiles are two units each, k-blocks [0, kb_half) and [kb_half, nkb)
  int full_units, tail_tiles, kb_half;
};

// DUAL: every k-block multiplies one A tile by two B tiles (B1 then B2) into
// the same accumulator, e.g. X^T by the hi and lo halves of a split operand, so
// that A is read once.
template <int BN, bool DUAL = false>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + (DUAL ? 2 : 1) * B_BYTES;
  // BN = 64 (the rank-r contractions) keeps 4 stages (3 when dual) so that two CTAs fit on an SM.
  static constexpr int STAGES =
      BN == 64 ? (DUAL ? 3 : 4) : ((200 * 1024) / STAGE_BYTES > 8 ? 8 : (200 * 1024) / STAGE_BYTES);
  static constexpr int TMEM_COLS = (2 * BN) < 32 ? 32 : 2 * BN;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;  // 128-byte swizzle
  return d;
}

constexpr uint32_t instr_desc(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                       // D format fp32
         | (1u << 7) | (1u << 10)        // A, B bf16
         | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16)
         | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Bounded wait that also gives up when another role has already aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              int32_t* err, int32_t code) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitBoundCycles) {
      report_error(err, code);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// wait_or_abort with acquire at cluster scope: for a barrier that threads of
// the peer CTA arrive on after writing their own shared memory, which the
// pair's MMAs then read.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool wait_or_abort_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                      int32_t* err, int32_t code) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitBoundCycles) {
      report_error(err, code);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// Tile (tm, tn) and k-block range of work unit `unit`. Consecutive units run
// at the same time on consecutive CTAs (pairs), so the order decides which A
// and B slabs are read from DRAM together: with bands of group_m M tiles the
// ~74 tiles in flight on 148 SMs cover about 8 x 9 tiles, so each wave reads
// about 17 slabs instead of the 16 + 5 of an M-fastest order.
__device__ __forceinline__ void decode_unit(const TileSched& ts, int unit, int& tm, int& tn, int& kb0, int& kb1) {
  int split = 0;
  if (ts.group_m > 0) {
    const int band = ts.group_m * ts.tiles_n;
    const int b = unit / band;
    const int first_m = b * ts.group_m;
    const int gm = min(ts.tiles_m - first_m, ts.group_m);
    const int r = unit - b * band;
    tm = first_m + r % gm;
    tn = r / gm;
  } else {
    tm = unit % ts.tiles_m;
    const int rest = unit / ts.tiles_m;
    tn = rest % ts.tiles_n;
    split = rest / ts.tiles_n;
  }
  kb0 = split * ts.kb_per_split;
  kb1 = min(ts.nkb, kb0 + ts.kb_per_split);
}

// Work unit of the 2-CTA kernels: tile (tm, tn), k-blocks [kb0, kb1), and for
// half a split tile its half (0, 1; -1 for a whole tile) and tail index.
__device__ __forceinline__ void decode_unit_pair(const TileSched& ts, int unit, int& tm, int& tn, int& kb0, int& kb1,
                                                 int& half, int& tail) {
  int t = unit;
  half = -1;
  tail = 0;
  if (unit >= ts.full_units) {
    const int v = unit - ts.full_units;
    tail = v >> 1;
    half = v & 1;
    t = ts.full_units + tail;
  }
  decode_unit(ts, t, tm, tn, kb0, kb1);
  if (half == 0) kb1 = ts.kb_half;
  if (half == 1) kb0 = ts.kb_half;
}

template <int BN, bool A_MN, bool B_MN, int OUT, bool DUAL = false>
__global__ void __launch_bounds__(kThreads)
k_tc_gemm(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
          const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2, TileSched ts,
          int M, int Nc, EpiParams ep, int32_t* err) {
  using C = Cfg<BN, DUAL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acce + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_units = ts.tiles_m * ts.tiles_n * ts.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA1);
    prefetch_tmap(&tmB1);
    prefetch_tmap(&tmA2);
    prefetch_tmap(&tmB2);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_enter();  // inputs written by the preceding kernel are visible from here on

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t outstanding = 0;      // stages loaded but not yet seen freed
      uint32_t out_parity = 0;       // parity each outstanding stage's load completes with
      bool ok = true;
      for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
        int tm, tn, kb0, kb1;
        decode_unit(ts, unit, tm, tn, kb0, kb1);
        const int m0 = tm * BM, n0 = tn * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort(&empty[stage], phase ^ 1u, abort_flag, err, DEV_TIMEOUT_SMEM_EMPTY)) {
            ok = false;
            break;
          }
          outstanding &= ~(1u << stage);
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          const bool slab = kb >= ts.nk1;
          const CUtensorMap* ta = slab ? &tmA2 : &tmA1;
          const CUtensorMap* tb = slab ? &tmB2 : &tmB1;
          const int k0 = (slab ? kb - ts.nk1 : kb) * BK;
          if (A_MN) {
            tma_load_2d(sa, ta, &full[stage], m0, k0);
            tma_load_2d(sa + 8192, ta, &full[stage], m0 + 64, k0);
          } else {
            tma_load_2d(sa, ta, &full[stage], k0, m0);
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) tma_load_2d(sb + j * 8192, tb, &full[stage], n0 + 64 * j, k0);
          } else {
            tma_load_2d(sb, tb, &full[stage], k0, n0);
          }
          if (DUAL) {  // the second B tile, same coordinates
            if (B_MN) {
#pragma unroll
              for (int j = 0; j < BN / 64; ++j)
                tma_load_2d(sb + C::B_BYTES + j * 8192, &tmB2, &full[stage], n0 + 64 * j, k0);
            } else {
              tma_load_2d(sb + C::B_BYTES, &tmB2, &full[stage], k0, n0);
            }
          }
          outstanding |= (1u << stage);
          out_parity = (out_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        for (int s = 0; s < C::STAGES; ++s)
          if (outstanding & (1u << s)) mbar_wait_bounded(&full[s], (out_parity >> s) & 1u, err, DEV_TIMEOUT_TMA_FULL);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
        int tm, tn, kb0, kb1;
        decode_unit(ts, unit, tm, tn, kb0, kb1);
        if (!wait_or_abort(&acce[acc], acc_phase ^ 1u, abort_flag, err, DEV_TIMEOUT_TMEM_EMPTY)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort(&full[stage], phase, abort_flag, err, DEV_TIMEOUT_TMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t da = A_MN ? smem_desc(sa + k * 2048, 8192, 1024) : smem_desc(sa + k * 32, 16, 1024);
            const uint64_t db = B_MN ? smem_desc(sb + k * 2048, 8192, 1024) : smem_desc(sb + k * 32, 16, 1024);
            mma_bf16(d_tmem, da, db, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
            if (DUAL) {
              const uint32_t sb2 = sb + C::B_BYTES;
              const uint64_t db2 =
                  B_MN ? smem_desc(sb2 + k * 2048, 8192, 1024) : smem_desc(sb2 + k * 32, 16, 1024);
              mma_bf16(d_tmem, da, db2, idesc, 1u);
            }
          }
          mma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&accf[acc]);       // accumulator ready for the epilogue
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
      int tm, tn, kb0, kb1;
      decode_unit(ts, unit, tm, tn, kb0, kb1);
      const int split = unit / (ts.tiles_m * ts.tiles_n);
      if (!wait_or_abort(&accf[acc], acc_phase, abort_flag, err, DEV_TIMEOUT_ACCUM)) break;
      tc_fence_after();
      const int row = tm * BM + row_in_tile;
      const bool row_ok = row < M;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN + c * 32),
                  v);
        const int col0 = tn * BN + c * 32;
        if (!row_ok) continue;
        if (OUT == OUT_BF16) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(ep.C) + static_cast<int64_t>(row) * ep.ldc + col0;
          if (col0 + 32 <= Nc && (ep.ldc % 8) == 0) {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              d4[q] = make_uint4(pack_bf16x2(v[8 * q + 0], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                 pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < Nc) dst[j] = __float2bfloat16_rn(v[j]);
          }
        } else if (OUT == OUT_LORA) {
          const int64_t po = static_cast<int64_t>(row) * ep.ld_pad + col0;
          uint4* sd = ep.s_bf16 ? reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(ep.s_bf16) + po) : nullptr;
          uint4* hd = ep.hi ? reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(ep.hi) + po) : nullptr;
          uint4* ld = ep.lo ? reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(ep.lo) + po) : nullptr;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t s4[4], h4[4], l4[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float a = v[8 * q + 2 * h], b = v[8 * q + 2 * h + 1];
              s4[h] = pack_bf16x2(ep.s * a, ep.s * b);
              h4[h] = pack_bf16x2(a, b);
              const float ah = bf16lo_to_f32(h4[h]), bh = bf16hi_to_f32(h4[h]);
              l4[h] = pack_bf16x2(a - ah, b - bh);
            }
            if (sd) sd[q] = make_uint4(s4[0], s4[1], s4[2], s4[3]);
            if (hd) hd[q] = make_uint4(h4[0], h4[1], h4[2], h4[3]);
            if (ld) ld[q] = make_uint4(l4[0], l4[1], l4[2], l4[3]);
          }
          if (ep.f32) {
            float* fd = ep.f32 + static_cast<int64_t>(row) * ep.ld_f32;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < Nc) fd[col0 + j] = v[j];
          }
        } else {  // OUT_PARTIAL
          float* pd = ep.P + (static_cast<int64_t>(split) * M + row) * Nc + col0;
          if (col0 + 32 <= Nc && (Nc % 4) == 0) {
            float4* p4 = reinterpret_cast<float4*>(pd);
#pragma unroll
            for (int q = 0; q < 8; ++q) p4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < Nc) pd[j] = v[j];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acce[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// 2-CTA variant for the large GEMMs: a cluster of two CTAs computes a 256x256
// tile with tcgen05.mma.cta_group::2 (M = 256 split 128/128 across the pair's
// tensor memories, B split 128/128 across their shared memories), so each SM
// streams 32 KB of operands per 64-deep k-block instead of 48 KB.
//   - Both CTAs load their halves with TMA; the loads complete on the even
//     (leader) CTA's full barrier, which the leader's producer arms with the
//     bytes of both halves.
//   - The leader's MMA thread issues the MMAs and commits with multicast to the
//     empty and accumulator-full barriers of both CTAs.
//   - Each CTA drains its own accumulator rows; both epilogues arrive on the
//     leader's accumulator-empty barrier (the odd CTA remotely).

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t map_to_cta(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const void* tmap, uint32_t bar_cluster_addr,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(bar_cluster_addr), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr) : "memory");
}

template <bool B_MN>
struct Cfg2 {
  static constexpr int A_BYTES = 128 * BK * 2;   // this CTA's half of A
  static constexpr int B_BYTES = 128 * BK * 2;   // this CTA's half of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = 6;
  static constexpr int TMEM_COLS = 512;          // two 256-column accumulators
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + 256;
};

// The tail of a pair GEMM's persistent schedule: when the last wave would leave
// at least half of the pairs idle, each of its tiles is split in two halves
// along K that run side by side. For each warp's 32 rows, each half writes its
// fp32 partial, then swaps the launch's tag into the rows' flag (acquire-
// release, GPU scope); the half that finds the tag already there adds the other
// partial to its own accumulator and writes C, then puts the flag back to
// another value, so that a replay of the same launch (a CUDA graph) starts
// clean. No half waits for the other, and own + other is the same sum in either
// order.
struct TailParams {
  float* part;               // fp32 [2 halves][kPairMaxTail][2 ranks][128 rows][256 cols]
  unsigned long long* flag;  // [kPairMaxTail][2 ranks][4 warps]
  unsigned long long tag;    // unique to the launch
};

__device__ __forceinline__ unsigned long long atom_exch_acq_rel_gpu(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.exch.acq_rel.gpu.global.b64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}

// Epilogue of one unit by one of warps 2..5 of a CTA of the pair (32 of the
// CTA's 128 rows of the 256 x 256 tile in accumulator `acc`): bf16 C, or for
// half a split tile the partial and, by the second half to arrive, the sum.
// AHEAD: load the other partial's next chunk while a chunk is summed (32 more
// registers; the NF4-decoding kernel, at 704 threads, has none to spare).
template <bool AHEAD>
__device__ __forceinline__ void pair_epilogue_unit(uint32_t tmem_base, int acc, int quarter, int lane, uint32_t rank,
                                                   int tm, int tn, int half, int tail, int M, int Nc,
                                                   const EpiParams& ep, const TailParams& tp) {
  constexpr int BN2 = 256;
  constexpr size_t kPart = 128 * 256;  // floats of one (half, tail, rank) partial
  const int row_in_tile = quarter * 32 + lane;
  const int row = tm * 256 + static_cast<int>(rank) * 128 + row_in_tile;
  const bool row_ok = row < M;
  const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN2);
  const float* other = nullptr;
  unsigned long long* flag = tp.flag + (static_cast<size_t>(tail) * 2 + rank) * 4 + quarter;
  if (half >= 0) {
    float* mine = tp.part + ((static_cast<size_t>(half) * kPairMaxTail + tail) * 2 + rank) * kPart +
                  static_cast<size_t>(row_in_tile) * BN2;
#pragma unroll 1
    for (int c = 0; c < BN2 / 32; ++c) {
      float v[32];
      tmem_ld32(tacc + static_cast<uint32_t>(c * 32), v);
      if (row_ok) {
        float4* d = reinterpret_cast<float4*>(mine + c * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q) __stcg(d + q, make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]));
      }
    }
    __syncwarp();  // the lanes' partial stores are ordered before lane 0's release below
    unsigned long long prev = 0;
    if (lane == 0) prev = atom_exch_acq_rel_gpu(flag, tp.tag);
    if (!__shfl_sync(0xffffffffu, prev == tp.tag ? 1 : 0, 0)) return;  // the other half finishes these rows
    __syncwarp();  // lane 0's acquire is ordered before every lane's reads of the other partial
    other = tp.part + ((static_cast<size_t>(1 - half) * kPairMaxTail + tail) * 2 + rank) * kPart +
            static_cast<size_t>(row_in_tile) * BN2;
  }
  float4 nxt[8];
  if (AHEAD && other && row_ok) {
#pragma unroll
    for (int q = 0; q < 8; ++q) nxt[q] = __ldcg(reinterpret_cast<const float4*>(other) + q);
  }
#pragma unroll 1
  for (int c = 0; c < BN2 / 32; ++c) {
    float v[32];
    tmem_ld32(tacc + static_cast<uint32_t>(c * 32), v);
    const int col0 = tn * BN2 + c * 32;
    if (!row_ok) continue;
    if (other) {
      float4 cur[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        cur[q] = AHEAD ? nxt[q] : __ldcg(reinterpret_cast<const float4*>(other + c * 32) + q);
      if (AHEAD && c + 1 < BN2 / 32) {
#pragma unroll
        for (int q = 0; q < 8; ++q) nxt[q] = __ldcg(reinterpret_cast<const float4*>(other + (c + 1) * 32) + q);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        v[4 * q] += cur[q].x;
        v[4 * q + 1] += cur[q].y;
        v[4 * q + 2] += cur[q].z;
        v[4 * q + 3] += cur[q].w;
      }
    }
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(ep.C) + static_cast<int64_t>(row) * ep.ldc + col0;
    if (col0 + 32 <= Nc && (ep.ldc % 8) == 0) {
      uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        d4[q] = make_uint4(pack_bf16x2(v[8 * q + 0], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                           pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < Nc) dst[j] = __float2bfloat16_rn(v[j]);
    }
  }
  if (half >= 0 && lane == 0) *flag = ~tp.tag;
}

template <bool B_MN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
k_tc_gemm2(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
           const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2, TileSched ts, int M,
           int Nc, EpiParams ep, int32_t* err, TailParams tp) {
  using C = Cfg2<B_MN>;
  constexpr int BN2 = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acce + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int n_units = ts.full_units + 2 * ts.tail_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 256);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA1);
    prefetch_tmap(&tmB1);
    prefetch_tmap(&tmA2);
    prefetch_tmap(&tmB2);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_enter();  // inputs written by the preceding kernel are visible from here on

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int unit = pair; unit < n_units && ok; unit += npairs) {
        int tm, tn, kb0, kb1, half, tail;
        decode_unit_pair(ts, unit, tm, tn, kb0, kb1, half, tail);
        const int m0 = tm * 256 + static_cast<int>(rank) * 128;
        const int n0 = tn * BN2 + static_cast<int>(rank) * 128;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort(&empty[stage], phase ^ 1u, abort_flag, err, DEV_TIMEOUT_SMEM_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          const uint32_t fbar = map_to_cta(smem_u32(&full[stage]), 0);
          const bool slab = kb >= ts.nk1;
          const CUtensorMap* ta = slab ? &tmA2 : &tmA1;
          const CUtensorMap* tb = slab ? &tmB2 : &tmB1;
          const int k0 = (slab ? kb - ts.nk1 : kb) * BK;
          tma_load_2d_pair(sa, ta, fbar, k0, m0);
          if (B_MN) {
            tma_load_2d_pair(sb, tb, fbar, n0, k0);
            tma_load_2d_pair(sb + 8192, tb, fbar, n0 + 64, k0);
          } else {
            tma_load_2d_pair(sb, tb, fbar, k0, n0);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA only) ----------------
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = instr_desc(256, BN2, false, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int unit = pair; unit < n_units && ok; unit += npairs) {
        int tm, tn, kb0, kb1, half, tail;
        decode_unit_pair(ts, unit, tm, tn, kb0, kb1, half, tail);
        if (!wait_or_abort(&acce[acc], acc_phase ^ 1u, abort_flag, err, DEV_TIMEOUT_TMEM_EMPTY)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN2);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort(&full[stage], phase, abort_flag, err, DEV_TIMEOUT_TMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t da = smem_desc(sa + k * 32, 16, 1024);
            const uint64_t db = B_MN ? smem_desc(sb + k * 2048, 8192, 1024) : smem_desc(sb + k * 32, 16, 1024);
            mma_bf16_pair(d_tmem, da, db, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(&accf[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5, both CTAs) ----------------
    const int quarter = warp & 3;
    const uint32_t acce_leader0 = map_to_cta(smem_u32(&acce[0]), 0);
    const uint32_t acce_leader1 = map_to_cta(smem_u32(&acce[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int unit = pair; unit < n_units; unit += npairs) {
      int tm, tn, kb0, kb1, half, tail;
      decode_unit_pair(ts, unit, tm, tn, kb0, kb1, half, tail);
      if (!wait_or_abort(&accf[acc], acc_phase, abort_flag, err, DEV_TIMEOUT_ACCUM)) break;
      tc_fence_after();
      pair_epilogue_unit<true>(tmem_base, acc, quarter, lane, rank, tm, tn, half, tail, M, Nc, ep, tp);
      tc_fence_before();
      mbar_arrive_cluster(acc ? acce_leader1 : acce_leader0);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Forward GEMM with the NF4 weight decoded into shared memory ("QLoRA vs
// ChatGPT", capability 5: the frozen weight is dequantized on the fly, block by
// block): C = X W'^T + [sT] B^T like k_tc_gemm2<false>, but the B stages of the
// main k-blocks are written by eight decoder warps per CTA from the packed
// codes and block constants (bit-identical W' to the standalone dequant), not
// loaded by TMA from a dequantized copy of W' in memory. A k-block of 64 is one
// 64-weight block of each weight row, so a lane pair decodes one row of a stage
// (32 weights each) from 16 bytes of codes and one constant, and stores the
// bf16 values in the 128-byte-swizzled K-major layout TMA would have written.
// The leader CTA's full barrier of a stage counts the producer's arrival (with
// the TMA bytes) and one arrival per decoder warp of both CTAs (the odd CTA's
// remotely); decoder warps fence their generic stores for the async proxy
// before arriving. The LoRA slab (sT against B) is TMA-loaded as before, and
// the decoder warps arrive on its stages without writing.

constexpr int kDecWarps = 8;     // decoder warps per group: one group fills one stage
constexpr int kDecGroups = 2;    // groups take alternate k-blocks
constexpr int kNf4Threads = kThreads + kDecGroups * kDecWarps * 32;

struct Nf4Src {
  const uint8_t* packed;
  const int8_t* q;
  const float* dqs;
  const float* mean;
  const float* absmax;   // single-level storage (q, dqs, mean unused) when not null
  int64_t N, K;
};

// B_MN = false: the forward, B = W' [N, K] (K-major): the CTA's row rl of a
// stage is weight row n0 + rl, block kb. B_MN = true: dX = dY W', B = W' with
// the contraction along its rows (MN-major, two 64-column boxes per stage): row
// rl of a stage is weight row 64 kb + (rl & 63), block column n0 / 64 + (rl >> 6).
// Either way the row's 128 bytes sit at rl * 128 with the same swizzle.
template <bool B_MN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kNf4Threads, 1)
k_tc_gemm2_nf4(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmA2,
               const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ Nf4Src src, TileSched ts, int M,
               int Nc, EpiParams ep, int32_t* err, const __grid_constant__ Nf4Codebook cb, TailParams tp) {
  using C = Cfg2<B_MN>;
  constexpr int BN2 = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acce + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int n_units = ts.full_units + 2 * ts.tail_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1 + 2 * kDecWarps);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 256);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA1);
    prefetch_tmap(&tmA2);
    prefetch_tmap(&tmB2);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_enter();  // inputs written by the preceding kernel are visible from here on

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs): A always, B only for the slab ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int unit = pair; unit < n_units && ok; unit += npairs) {
        int tm, tn, kb0, kb1, half, tail;
        decode_unit_pair(ts, unit, tm, tn, kb0, kb1, half, tail);
        const int m0 = tm * 256 + static_cast<int>(rank) * 128;
        const int n0 = tn * BN2 + static_cast<int>(rank) * 128;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort(&empty[stage], phase ^ 1u, abort_flag, err, DEV_TIMEOUT_SMEM_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          const bool slab = kb >= ts.nk1;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (slab ? C::STAGE_BYTES : C::A_BYTES));
          const uint32_t fbar = map_to_cta(smem_u32(&full[stage]), 0);
          const int k0 = (slab ? kb - ts.nk1 : kb) * BK;
          tma_load_2d_pair(sa, slab ? &tmA2 : &tmA1, fbar, k0, m0);
          if (slab) {
            if (B_MN) {
              tma_load_2d_pair(sb, &tmB2, fbar, n0, k0);
              tma_load_2d_pair(sb + 8192, &tmB2, fbar, n0 + 64, k0);
            } else {
              tma_load_2d_pair(sb, &tmB2, fbar, k0, n0);
            }
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA only) ----------------
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = instr_desc(256, BN2, false, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int unit = pair; unit < n_units && ok; unit += npairs) {
        int tm, tn, kb0, kb1, half, tail;
        decode_unit_pair(ts, unit, tm, tn, kb0, kb1, half, tail);
        if (!wait_or_abort(&acce[acc], acc_phase ^ 1u, abort_flag, err, DEV_TIMEOUT_TMEM_EMPTY)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN2);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort_cluster(&full[stage], phase, abort_flag, err, DEV_TIMEOUT_TMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t da = smem_desc(sa + k * 32, 16, 1024);
            const uint64_t db = B_MN ? smem_desc(sb + k * 2048, 8192, 1024) : smem_desc(sb + k * 32, 16, 1024);
            mma_bf16_pair(d_tmem, da, db, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(&accf[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else if (warp < 6) {
    // ---------------- epilogue (warps 2..5, both CTAs) ----------------
    const int quarter = warp & 3;
    const uint32_t acce_leader0 = map_to_cta(smem_u32(&acce[0]), 0);
    const uint32_t acce_leader1 = map_to_cta(smem_u32(&acce[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int unit = pair; unit < n_units; unit += npairs) {
      int tm, tn, kb0, kb1, half, tail;
      decode_unit_pair(ts, unit, tm, tn, kb0, kb1, half, tail);
      if (!wait_or_abort(&accf[acc], acc_phase, abort_flag, err, DEV_TIMEOUT_ACCUM)) break;
      tc_fence_after();
      pair_epilogue_unit<false>(tmem_base, acc, quarter, lane, rank, tm, tn, half, tail, M, Nc, ep, tp);
      tc_fence_before();
      mbar_arrive_cluster(acc ? acce_leader1 : acce_leader0);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  } else {
    // ---------------- decoder warps (6..13, both CTAs) ----------------
    // lanes 2i and 2i + 1 of decoder warp d write row 16 d + i of the CTA's
    // 128 B rows, weights 32 h .. 32 h + 31 (h = lane & 1) of the k-block
    const int dw = (warp - 6) % kDecWarps;
    const int group = (warp - 6) / kDecWarps;
    const int rl = dw * 16 + (lane >> 1);
    const int h = lane & 1;
    const int64_t nkb = src.K / 64;
    const bool single = src.absmax != nullptr;
    const float mu = single ? 0.0f : __ldg(src.mean);
    const uint32_t leader_full0 = map_to_cta(smem_u32(&full[0]), 0);
    const uint32_t swz = static_cast<uint32_t>(rl & 7);
    int stage = 0;
    uint32_t phase = 0;
    uint32_t it = 0;  // k-blocks so far (all units): group it % kDecGroups fills this one
    bool ok = true;
    for (int unit = pair; unit < n_units && ok; unit += npairs) {
      int tm, tn, kb0, kb1, half, tail;
      decode_unit_pair(ts, unit, tm, tn, kb0, kb1, half, tail);
      const int64_t n0 = static_cast<int64_t>(tn) * BN2 + static_cast<int64_t>(rank) * 128;
      // codes and constant of the first main k-block of the tile, then one ahead
      uint4 cur = make_uint4(0u, 0u, 0u, 0u);
      float mcur = 0.0f;
      auto fetch = [&](int kb, uint4& c, float& mval) {
        const int64_t wrow = B_MN ? static_cast<int64_t>(kb) * 64 + (rl & 63) : n0 + rl;
        const int64_t bcol = B_MN ? n0 / 64 + (rl >> 6) : kb;
        if (kb >= ts.nk1 || wrow >= src.N || bcol >= nkb) {
          c = make_uint4(0u, 0u, 0u, 0u);
          mval = 0.0f;
          return;
        }
        const int64_t b = wrow * nkb + bcol;
        c = __ldg(reinterpret_cast<const uint4*>(src.packed + b * 32) + h);  // reused by every M tile: keep in L2
        mval = single ? __ldg(src.absmax + b)
                      : __fmaf_rn(static_cast<float>(__ldg(src.q + b)), __ldg(src.dqs + (b >> 8)), mu);
      };
      // this group's first k-block of the unit
      int kbg = kb0 + static_cast<int>((static_cast<uint32_t>(group) - it) % kDecGroups);
      fetch(kbg, cur, mcur);
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        if (static_cast<int>(it % kDecGroups) != group) {  // the other group's stage
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          continue;
        }
        uint4 nxt;
        float mnxt;
        fetch(kb + kDecGroups < kb1 ? kb + kDecGroups : kb1, nxt, mnxt);
        if (!wait_or_abort(&empty[stage], phase ^ 1u, abort_flag, err, DEV_TIMEOUT_SMEM_EMPTY)) {
          ok = false;
          break;
        }
        if (kb < ts.nk1) {
          // decode 32 weights: bf16_rn(codebook[code] * m') for the codes of this row
          const Nf4Lut t = make_nf4_lut(cb, mcur);
          uint32_t o[16];
          nf4_lookup8(t, cur.x, o + 0);
          nf4_lookup8(t, cur.y, o + 4);
          nf4_lookup8(t, cur.z, o + 8);
          nf4_lookup8(t, cur.w, o + 12);
          uint8_t* rowp = smem + stage * C::STAGE_BYTES + C::A_BYTES + rl * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {  // 16-byte chunk 4 h + q of the row, 128-byte swizzle
            const uint32_t chunk = (static_cast<uint32_t>(4 * h + q) ^ swz) * 16u;
            *reinterpret_cast<uint4*>(rowp + chunk) = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          }
          // the tensor core reads the stage through the async proxy
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(leader_full0 + static_cast<uint32_t>(stage) * 8u);
        cur = nxt;
        mcur = mnxt;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// host side

// 2-D bf16 tensor [outer, inner] with row stride ld (elements); box {64, box_outer}.
bool make_map(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld, int box_outer) {
  PFN_encodeTiled enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Operand description for the host launcher.
struct Operand {
  const void* p;
  int64_t rows_mn;   // extent along the GEMM's M (for A) or N (for B)
  int64_t k;         // extent along the reduction
  int64_t ld;        // row stride in elements of the stored matrix
  bool mn_major;     // stored [k, mn] (mn contiguous) instead of [mn, k]
};

bool map_operand(CUtensorMap* m, const Operand& o, int tile_mn) {
  if (o.mn_major) return make_map(m, o.p, o.rows_mn, o.k, o.ld, 64);
  return make_map(m, o.p, o.k, o.rows_mn, o.ld, tile_mn);
}

template <int BN, bool A_MN, bool B_MN, int OUT, bool DUAL = false>
cudaError_t run(const Operand& a1, const Operand& b1, const Operand* a2, const Operand* b2, int M, int Nc,
                int splits, const EpiParams& ep, int num_sms, int32_t* err, cudaStream_t stream) {
  using C = Cfg<BN, DUAL>;
  CUtensorMap ta1, tb1, ta2, tb2;
  if (!map_operand(&ta1, a1, BM) || !map_operand(&tb1, b1, BN)) return cudaErrorInvalidValue;
  if (a2 && b2) {
    if (!map_operand(&ta2, *a2, BM) || !map_operand(&tb2, *b2, BN)) return cudaErrorInvalidValue;
  } else {
    ta2 = ta1;
    tb2 = tb1;
  }
  TileSched ts{};  // group_m = 0: M-fastest
  ts.tiles_m = static_cast<int>((M + BM - 1) / BM);
  ts.tiles_n = static_cast<int>((Nc + BN - 1) / BN);
  ts.nk1 = static_cast<int>((a1.k + BK - 1) / BK);
  // DUAL: b2 is the second B operand of every k-block, not a slab of its own
  const int nk2 = (a2 && b2 && !DUAL) ? static_cast<int>((a2->k + BK - 1) / BK) : 0;
  ts.nkb = ts.nk1 + nk2;
  // callers pass a count from split_count(), so every piece is non-empty and the
  // number of partial slices written equals `splits`
  if (splits != split_count(ts.nkb, splits)) return cudaErrorInvalidValue;
  ts.kb_per_split = (ts.nkb + splits - 1) / splits;
  ts.splits = splits;
  const int units = ts.tiles_m * ts.tiles_n * ts.splits;
  const int slots = (BN == 64 ? 2 : 1) * num_sms;  // resident CTAs
  const int grid = units < slots ? units : slots;
  auto kern = k_tc_gemm<BN, A_MN, B_MN, OUT, DUAL>;
  const cudaError_t e = ensure_smem_limit<k_tc_gemm<BN, A_MN, B_MN, OUT, DUAL>>(C::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(kThreads), C::SMEM, stream, ta1, tb1, ta2, tb2, ts, M, Nc, ep, err);
}

// Units and pairs of a 2-CTA GEMM (ts.tiles_m, tiles_n, nkb set): whole tiles,
// and when the last wave would leave at least half of the pairs idle and the
// reduction is long, its tiles split in two along K (both halves then run in
// that wave).
int plan_pair_units(TileSched& ts, int num_sms, bool can_split) {
  const int tiles = ts.tiles_m * ts.tiles_n;
  int pairs = num_sms / 2;
  if (pairs < 1) pairs = 1;
  const int rem = tiles % pairs;
  ts.full_units = tiles;
  ts.tail_tiles = 0;
  ts.kb_half = ts.nkb;
  // (halves of fewer than ~48 k-blocks measured slower: the split tile's
  // epilogue outweighs half a short tile; 4096x4096 at M = 4096: 118 -> 126 us)
  if (can_split && rem > 0 && 2 * rem <= pairs && rem <= kPairMaxTail && ts.nkb >= 96) {
    ts.full_units = tiles - rem;
    ts.tail_tiles = rem;
    ts.kb_half = (ts.nkb + 1) / 2;
  }
  const int units = ts.full_units + 2 * ts.tail_tiles;
  return pairs < units ? pairs : units;
}

// A tag unique to each launch of a 2-CTA GEMM (the tail's flags compare
// against it): a 64-bit counter from a random start.
unsigned long long next_pair_tag() {
  static std::atomic<unsigned long long> counter{[] {
    std::random_device rd;
    return (static_cast<unsigned long long>(rd()) << 32) ^ static_cast<unsigned long long>(rd());
  }()};
  return counter.fetch_add(1, std::memory_order_relaxed);
}

TailParams tail_params(void* tail_ws) {
  TailParams tp{};
  if (tail_ws) {
    tp.part = static_cast<float*>(tail_ws);
    tp.flag = reinterpret_cast<unsigned long long*>(static_cast<char*>(tail_ws) +
                                                   static_cast<size_t>(kPairMaxTail) * 2 * 2 * 128 * 256 * sizeof(float));
    tp.tag = next_pair_tag();
  }
  return tp;
}

template <bool B_MN>
cudaError_t run_pair(const Operand& a1, const Operand& b1, const Operand& a2, const Operand& b2, int M, int Nc,
                     const EpiParams& ep, void* tail_ws, int num_sms, int32_t* err, cudaStream_t stream) {
  using C = Cfg2<B_MN>;
  CUtensorMap ta1, tb1, ta2, tb2;
  // each CTA loads 128 rows of A and 128 of B's output dimension per box
  if (!map_operand(&ta1, a1, 128) || !map_operand(&tb1, b1, 128)) return cudaErrorInvalidValue;
  if (!map_operand(&ta2, a2, 128) || !map_operand(&tb2, b2, 128)) return cudaErrorInvalidValue;
  TileSched ts{};
  // dX (MN-major B): bands of 8 M tiles cut its DRAM reads (465 -> 416 MB on
  // 11008x4096, M = 4096); the forward keeps the M-fastest order, which reads
  // W' once (141 MB against 220 MB banded)
  ts.group_m = B_MN ? 8 : 0;
  ts.tiles_m = static_cast<int>((M + 255) / 256);
  ts.tiles_n = static_cast<int>((Nc + 255) / 256);
  ts.nk1 = static_cast<int>((a1.k + BK - 1) / BK);
  ts.nkb = ts.nk1 + static_cast<int>((a2.k + BK - 1) / BK);
  ts.splits = 1;
  ts.kb_per_split = ts.nkb;
  const int pairs = plan_pair_units(ts, num_sms, tail_ws != nullptr);
  auto kern = k_tc_gemm2<B_MN>;
  const cudaError_t e = ensure_smem_limit<k_tc_gemm2<B_MN>>(C::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(2 * pairs), dim3(kThreads), C::SMEM, stream, ta1, tb1, ta2, tb2, ts, M, Nc, ep, err,
                    tail_params(tail_ws));
}

}  // namespace

// The 2-CTA kernel serves the large GEMMs (M >= 256 tokens); QLORA_TC_PAIR=0 in
// the environment selects the 1-CTA kernel instead (for comparisons).
bool use_pair_kernel(int64_t M) {
  static const bool enabled = [] {
    const char* e = std::getenv("QLORA_TC_PAIR");
    return !(e && e[0] == '0');
  }();
  return enabled && M >= 256;
}

// Forward main GEMM: Y[M,N] = X[M,K] W'[N,K]^T + sT[M,rpad] Bl[N,r]^T
cudaError_t launch_gemm_fwd(const void* X, const void* Wd, const void* sT, const void* Bl, int64_t M, int64_t N,
                            int64_t K, int r, int rpad, void* Y, void* tail_ws, int num_sms, int32_t* err,
                            cudaStream_t stream) {
  Operand a1{X, M, K, K, false}, b1{Wd, N, K, K, false};
  Operand a2{sT, M, rpad, rpad, false}, b2{Bl, N, r, r, false};
  EpiParams ep{};
  ep.C = Y;
  ep.ldc = N;
  if (use_pair_kernel(M))
    return run_pair<false>(a1, b1, a2, b2, static_cast<int>(M), static_cast<int>(N), ep, tail_ws, num_sms, err,
                           stream);
  return run<256, false, false, OUT_BF16>(a1, b1, &a2, &b2, static_cast<int>(M), static_cast<int>(N), 1, ep,
                                          num_sms, err, stream);
}

// GEMMs with W' decoded from NF4 inside the 2-CTA kernel (M >= 256):
// forward Y[M,N] = X[M,K] dequant(w)^T + sT[M,rpad] Bl[N,r]^T (B_MN false), and
// dX[M,K] = dY[M,N] dequant(w) + sU[M,rpad] Al[r,K] (B_MN true).
template <bool B_MN>
cudaError_t run_pair_nf4(const void* A1, int64_t K1, const Nf4View& w, const void* s_lora, const void* lora_w,
                         int64_t M, int r, int rpad, void* out, void* tail_ws, const float codebook[16], int num_sms,
                         int32_t* err, cudaStream_t stream) {
  using C = Cfg2<B_MN>;
  const int64_t N = w.N, K = w.K;
  const int64_t Nc = B_MN ? K : N;  // output columns
  Operand a1{A1, M, K1, K1, false};
  Operand a2{s_lora, M, rpad, rpad, false};
  Operand b2 = B_MN ? Operand{lora_w, K, r, K, true} : Operand{lora_w, N, r, r, false};
  CUtensorMap ta1, ta2, tb2;
  if (!map_operand(&ta1, a1, 128) || !map_operand(&ta2, a2, 128) || !map_operand(&tb2, b2, 128))
    return cudaErrorInvalidValue;
  TileSched ts{};
  // dX (MN-major B): bands of 8 M tiles cut its DRAM reads (465 -> 416 MB on
  // 11008x4096, M = 4096); the forward keeps the M-fastest order, which reads
  // W' once (141 MB against 220 MB banded)
  ts.group_m = B_MN ? 8 : 0;
  ts.tiles_m = static_cast<int>((M + 255) / 256);
  ts.tiles_n = static_cast<int>((Nc + 255) / 256);
  ts.nk1 = static_cast<int>((K1 + BK - 1) / BK);
  ts.nkb = ts.nk1 + static_cast<int>((rpad + BK - 1) / BK);
  ts.splits = 1;
  ts.kb_per_split = ts.nkb;
  const int pairs = plan_pair_units(ts, num_sms, tail_ws != nullptr);
  Nf4Src src{w.packed, w.absmax_q, w.dq_scale, w.mean, w.absmax, N, K};
  Nf4Codebook cb;
  for (int i = 0; i < 16; ++i) cb.c[i] = codebook[i];
  EpiParams ep{};
  ep.C = out;
  ep.ldc = Nc;
  const cudaError_t e = ensure_smem_limit<k_tc_gemm2_nf4<B_MN>>(C::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_tc_gemm2_nf4<B_MN>, dim3(2 * pairs), dim3(kNf4Threads), C::SMEM, stream, ta1, ta2, tb2, src,
                    ts, static_cast<int>(M), static_cast<int>(Nc), ep, err, cb, tail_params(tail_ws));
}

cudaError_t launch_gemm_fwd_nf4(const void* X, const Nf4View& w, const void* sT, const void* Bl, int64_t M, int r,
                                int rpad, void* Y, void* tail_ws, const float codebook[16], int num_sms, int32_t* err,
                                cudaStream_t stream) {
  return run_pair_nf4<false>(X, w.K, w, sT, Bl, M, r, rpad, Y, tail_ws, codebook, num_sms, err, stream);
}

cudaError_t launch_gemm_dx_nf4(const void* dY, const Nf4View& w, const void* sU, const void* Al, int64_t M, int r,
                               int rpad, void* dX, void* tail_ws, const float codebook[16], int num_sms, int32_t* err,
                               cudaStream_t stream) {
  return run_pair_nf4<true>(dY, w.N, w, sU, Al, M, r, rpad, dX, tail_ws, codebook, num_sms, err, stream);
}

// Backward dX: dX[M,K] = dY[M,N] W'[N,K] + sU[M,rpad] A[r,K]
cudaError_t launch_gemm_dx(const void* dY, const void* Wd, const void* sU, const void* Al, int64_t M, int64_t N,
                           int64_t K, int r, int rpad, void* dX, void* tail_ws, int num_sms, int32_t* err,
                           cudaStream_t stream) {
  Operand a1{dY, M, N, N, false}, b1{Wd, K, N, K, true};
  Operand a2{sU, M, rpad, rpad, false}, b2{Al, K, r, K, true};
  EpiParams ep{};
  ep.C = dX;
  ep.ldc = K;
  if (use_pair_kernel(M))
    return run_pair<true>(a1, b1, a2, b2, static_cast<int>(M), static_cast<int>(K), ep, tail_ws, num_sms, err,
                          stream);
  return run<256, false, true, OUT_BF16>(a1, b1, &a2, &b2, static_cast<int>(M), static_cast<int>(K), 1, ep,
                                         num_sms, err, stream);
}

// LoRA down projection, split over K: P[split][M][rpad] = partial sums of
// X[M,K] A[r,K]^T (columns >= r are zero); launch_lora_finish turns them into
// T (fp32, optional), sT = bf16(s T), T_hi = bf16(T), T_lo = bf16(T - T_hi).
cudaError_t launch_gemm_lora_t(const void* X, const void* Al, int64_t M, int64_t K, int r, int rpad, float* P,
                               int splits, int num_sms, int32_t* err, cudaStream_t stream) {
  Operand a1{X, M, K, K, false}, b1{Al, r, K, K, false};
  EpiParams ep{};
  ep.P = P;
  return run<64, false, false, OUT_PARTIAL>(a1, b1, nullptr, nullptr, static_cast<int>(M), rpad, splits, ep,
                                            num_sms, err, stream);
}

// LoRA up-gradient, split over N: P[split][M][rpad] = partial sums of dY[M,N] B[N,r].
cudaError_t launch_gemm_lora_u(const void* dY, const void* Bl, int64_t M, int64_t N, int r, int rpad, float* P,
                               int splits, int num_sms, int32_t* err, cudaStream_t stream) {
  Operand a1{dY, M, N, N, false}, b1{Bl, r, N, r, true};
  EpiParams ep{};
  ep.P = P;
  return run<64, false, true, OUT_PARTIAL>(a1, b1, nullptr, nullptr, static_cast<int>(M), rpad, splits, ep,
                                           num_sms, err, stream);
}

// Split reduction over tokens: P[split][R][rpad] = sum_m Q[m, R]^T (hi + lo)[m, rpad]
// with Q bf16 [M, R] (X for dA^T, dY for dB) and hi/lo bf16 [M, rpad].
cudaError_t launch_gemm_lora_grad(const void* Q, int64_t R, const void* hi, const void* lo, int64_t M, int rpad,
                                  float* P, int splits, int num_sms, int32_t* err, cudaStream_t stream) {
  // Q^T [R, M] times hi and lo [M, rpad]: each k-block of Q is read once and
  // multiplied by both halves
  Operand a1{Q, R, M, R, true}, b1{hi, rpad, M, rpad, true};
  Operand b2{lo, rpad, M, rpad, true};
  EpiParams ep{};
  ep.P = P;
  return run<64, true, true, OUT_PARTIAL, true>(a1, b1, &a1, &b2, static_cast<int>(R), rpad, splits, ep, num_sms,
                                                err, stream);
}

}  // namespace qlora
