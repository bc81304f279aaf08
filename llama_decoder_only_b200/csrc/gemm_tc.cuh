// bf16 projection / FFN GEMMs on the 5th-generation tensor cores (tcgen05).
//
// C = A · B^T with A [rows, K] and B [n, K] both K-major bf16, fp32
// accumulation in TMEM ([DeepDive] LLaMAAttention / LLaMAMLP: every Linear is
// y = x W^T with W [out, in]).  One CTA per SM, 6 warps:
//   warp 0      TMA producer (one elected lane): A and B tiles into a ring of
//               STAGES shared-memory stages, 128-byte swizzle, no multicast;
//   warp 1      TMEM allocator and MMA issuer (one lane): 4 x tcgen05.mma
//               (M=128, N=BN, K=16) per 64-wide k-block, commit frees the stage;
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (one TMEM lane = one
//               output row per thread; two warps per lane quadrant, each
//               taking half of the tile's columns), fused epilogue, global
//               store.
// The accumulator is double-buffered in TMEM (2 x BN fp32 columns), so the
// epilogue of one tile overlaps the main loop of the next.
//
// Two schedules:
//  * tile mode (prefill, SWAP = false): A = activations (tokens x K),
//    B = weight rows; persistent CTAs walk the (m-tile, n-tile) grid with the
//    m index fastest so concurrently running CTAs share weight tiles in L2.
//    Epilogues: bf16 store (QKV), fp32 residual add (o_proj, down), paired
//    SiLU(gate)·up with gate rows and up rows loaded into the two halves of
//    one B tile (gate_up), fp32 store (lm_head).
//  * stream-K mode (decode, SWAP = true): the weight is A (its rows fill the
//    MMA's M = 128) and the few token rows are B (N = BN >= tokens), so the
//    weight streams from HBM once.  The (weight tile, k-block) units are split
//    evenly over the CTAs; each CTA writes one fp32 partial per tile piece and
//    a separate reduce kernel adds the pieces in CTA order (deterministic)
//    and applies the epilogue.
//
// The weight can be given as up to three row segments with their own tensor
// maps (q, k, v when the three projections are not contiguous; gate and up).
#pragma once

#include "common.cuh"

namespace llama {

enum GemmEpi : int { EPI_BF16 = 0, EPI_RESID_F32 = 1, EPI_SWIGLU_BF16 = 2, EPI_F32 = 3, EPI_PARTIAL = 4 };

struct GemmParams {
  int K;
  int num_kb;          // ceil(K / 64)
  int act_rows;        // token rows of the activation operand
  int m_tiles;         // tile mode: ceil(act_rows / 128)
  int n_tiles;         // weight tiles over all segments
  int nseg;
  int seg_rows[3];     // weight rows per segment
  int seg_tile0[4];    // first weight tile of each segment (cumulative, [nseg] = n_tiles)
  int seg_col0[3];     // output column of each segment's row 0
  // epilogue (tile mode)
  void* out;
  int ldo;
  const float* resid;
  int ldr;
  // stream-K mode
  float* partial;
  long long units;     // n_tiles * num_kb
  int max_pieces;      // partial slots per CTA
  DevStatus* status;
  unsigned long long limit_ns;
};

constexpr int GEMM_EPI_WARPS = 8;
constexpr int GEMM_THREADS = 64 + 32 * GEMM_EPI_WARPS;

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = (200 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                        : (2 * BN <= 256) ? 256 : 512;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
};

// Work item shared by the three roles: one output tile and a k-block range.
struct GemmItem {
  int tile;   // tile mode: linear (m fastest); stream-K: weight tile
  int kb0, kb1;
  int slot;   // swap stream-K: partial slot within the CTA
};

struct GemmIter {
  // tile mode
  int next_tile, tile_count;
  // stream-K mode
  long long u, u1;
  int first_tile;
  int num_kb;
  bool streamk;

  __device__ void init(const GemmParams& p, bool sk) {
    streamk = sk;
    num_kb = p.num_kb;
    if (!sk) {
      next_tile = blockIdx.x;
      tile_count = p.m_tiles * p.n_tiles;
    } else {
      const long long G = gridDim.x;
      u = p.units * (long long)blockIdx.x / G;
      u1 = p.units * (long long)(blockIdx.x + 1) / G;
      first_tile = (int)(u / num_kb);
    }
  }
  __device__ bool next(GemmItem& it) {
    if (!streamk) {
      if (next_tile >= tile_count) return false;
      it.tile = next_tile;
      it.kb0 = 0;
      it.kb1 = num_kb;
      it.slot = 0;
      next_tile += gridDim.x;
      return true;
    }
    if (u >= u1) return false;
    it.tile = (int)(u / num_kb);
    it.kb0 = (int)(u % num_kb);
    long long rem = u1 - u;
    it.kb1 = (int)((long long)it.kb0 + rem < num_kb ? it.kb0 + rem : num_kb);
    it.slot = it.tile - first_tile;
    u += it.kb1 - it.kb0;
    return true;
  }
};

__device__ __forceinline__ int seg_of_tile(const GemmParams& p, int wtile) {
  int s = 0;
  if (p.nseg > 1 && wtile >= p.seg_tile0[1]) s = 1;
  if (p.nseg > 2 && wtile >= p.seg_tile0[2]) s = 2;
  return s;
}

template <int BN, bool SWAP, int EPI>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmAct, const __grid_constant__ CUtensorMap tmW0,
                   const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2,
                   const GemmParams p) {
  using C = GemmCfg<BN>;
  constexpr int STAGES = C::STAGES;
  constexpr int WROWS = SWAP ? 128 : BN;  // weight rows per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);

  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 32 * GEMM_EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmAct);
    tma_prefetch_desc(&tmW0);
    if (p.nseg > 1) tma_prefetch_desc(&tmW1);
    if (p.nseg > 2) tma_prefetch_desc(&tmW2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem_base = tmem_base_sh;
  WaitCtx wc{&abort_sh, p.status, p.limit_ns, SWAP ? 2 : 1};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int filled_parity[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) filled_parity[s] = -1;
      GemmIter it;
      it.init(p, SWAP);
      GemmItem item;
      bool ok = true;
      while (ok && it.next(item)) {
        int wtile, m0 = 0;
        if (SWAP) {
          wtile = item.tile;
        } else {
          wtile = item.tile / p.m_tiles;
          m0 = (item.tile % p.m_tiles) * 128;
        }
        const int seg = seg_of_tile(p, wtile);
        const int wrow0 = (wtile - p.seg_tile0[seg]) * WROWS;
        const CUtensorMap* wm = seg == 0 ? &tmW0 : (seg == 1 ? &tmW1 : &tmW2);
        for (int kb = item.kb0; kb < item.kb1; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc, 1)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
          mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
          if (SWAP) {
            tma_load_2d(sa, wm, full_bar(stage), kb * 64, wrow0);
            tma_load_2d(sb, &tmAct, full_bar(stage), kb * 64, 0);
          } else {
            tma_load_2d(sa, &tmAct, full_bar(stage), kb * 64, m0);
            if (EPI == EPI_SWIGLU_BF16) {
              // gate rows into the first half of the B tile, up rows into the second
              const int r0 = (wtile)*(BN / 2);
              tma_load_2d(sb, &tmW0, full_bar(stage), kb * 64, r0);
              tma_load_2d(sb + (BN / 2) * 128, &tmW1, full_bar(stage), kb * 64, r0);
            } else {
              tma_load_2d(sb, wm, full_bar(stage), kb * 64, wrow0);
            }
          }
          filled_parity[stage] = (int)phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // drain: every issued fill must have landed before the CTA may exit
      for (int s = 0; s < STAGES; ++s)
        if (filled_parity[s] >= 0) mbar_wait(full_bar(s), (uint32_t)filled_parity[s], wc, 9, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, 0, 0);
      int stage = 0;
      uint32_t phase = 0;
      int abuf = 0;
      uint32_t aphase = 0;
      bool issued = false;
      GemmIter it;
      it.init(p, SWAP);
      GemmItem item;
      bool ok = true;
      while (ok && it.next(item)) {
        if (!mbar_wait(acce_bar(abuf), aphase ^ 1u, wc, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * BN);
        for (int kb = item.kb0; kb < item.kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, wc, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = smem_desc_sw128(sa + k * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sb + k * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, IDESC, (kb > item.kb0 || k > 0) ? 1u : 0u);
          }
          issued = true;
          umma_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(accf_bar(abuf));
        if (++abuf == 2) {
          abuf = 0;
          aphase ^= 1u;
        }
      }
      if (issued) {
        // all MMAs of this thread complete before TMEM is released
        umma_commit(drain_bar);
        mbar_wait(drain_bar, 0, wc, 8, false);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may read
    const int half = (warp - 2) >> 2;          // which half of the tile's columns
    const int row = quad * 32 + lane;  // TMEM lane == accumulator row
    int abuf = 0;
    uint32_t aphase = 0;
    GemmIter it;
    it.init(p, SWAP);
    GemmItem item;
    while (it.next(item)) {
      if (!__all_sync(0xffffffffu, mbar_wait(accf_bar(abuf), aphase, wc, 4))) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(abuf * BN);
      if (SWAP) {
        // partial[(cta * max_pieces + slot)][token][128] (fp32); row = weight row in tile
        float* dst = p.partial + ((size_t)blockIdx.x * p.max_pieces + item.slot) * (size_t)BN * 128;
#pragma unroll 1
        for (int c = half * 16; c < BN; c += 32) {
          float v[16];
          tmem_ld16(tbase + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c + j < p.act_rows) dst[(size_t)(c + j) * 128 + row] = v[j];
        }
      } else {
        const int wtile = item.tile / p.m_tiles;
        const int m = (item.tile % p.m_tiles) * 128 + row;
        const bool row_ok = m < p.act_rows;

        if (EPI == EPI_SWIGLU_BF16) {
          const int n0 = wtile * (BN / 2);
          const int nlim = p.seg_rows[0];
          __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)m * p.ldo;
#pragma unroll 1
          for (int c = half * (BN / 4); c < (half + 1) * (BN / 4); c += 32) {
            float g[32], u[32];
            tmem_ld32(tbase + c, g);
            tmem_ld32(tbase + BN / 2 + c, u);
            tmem_ld_wait();
            if (row_ok) {
              const int n = n0 + c;
              if (n + 32 <= nlim) {
                uint4* o4 = reinterpret_cast<uint4*>(o + n);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  uint4 w;
                  w.x = pack_bf16x2(silu_f(g[8 * q + 0]) * u[8 * q + 0], silu_f(g[8 * q + 1]) * u[8 * q + 1]);
                  w.y = pack_bf16x2(silu_f(g[8 * q + 2]) * u[8 * q + 2], silu_f(g[8 * q + 3]) * u[8 * q + 3]);
                  w.z = pack_bf16x2(silu_f(g[8 * q + 4]) * u[8 * q + 4], silu_f(g[8 * q + 5]) * u[8 * q + 5]);
                  w.w = pack_bf16x2(silu_f(g[8 * q + 6]) * u[8 * q + 6], silu_f(g[8 * q + 7]) * u[8 * q + 7]);
                  o4[q] = w;
                }
              } else {
                for (int j = 0; j < 32; ++j)
                  if (n + j < nlim) o[n + j] = __float2bfloat16_rn(silu_f(g[j]) * u[j]);
              }
            }
          }
        } else {
          const int seg = seg_of_tile(p, wtile);
          const int nl0 = (wtile - p.seg_tile0[seg]) * BN;  // row within the segment
          const int nlim = p.seg_rows[seg];
          const int col0 = p.seg_col0[seg] + nl0;
#pragma unroll 1
          for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 32) {
            float v[32];
            tmem_ld32(tbase + c, v);
            tmem_ld_wait();
            if (!row_ok || nl0 + c >= nlim) continue;
            const bool full = nl0 + c + 32 <= nlim;
            const int n = col0 + c;
            if (EPI == EPI_BF16) {
              __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)m * p.ldo + n;
              if (full) {
                uint4* o4 = reinterpret_cast<uint4*>(o);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  uint4 w;
                  w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
                  w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
                  w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
                  w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
                  o4[q] = w;
                }
              } else {
                for (int j = 0; j < 32 && nl0 + c + j < nlim; ++j) o[j] = __float2bfloat16_rn(v[j]);
              }
            } else if (EPI == EPI_RESID_F32) {
              float* o = reinterpret_cast<float*>(p.out) + (size_t)m * p.ldo + n;
              const float* r = p.resid + (size_t)m * p.ldr + n;
              if (full) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                  float4 rr = reinterpret_cast<const float4*>(r)[q];
                  float4 w = make_float4(rr.x + v[4 * q + 0], rr.y + v[4 * q + 1], rr.z + v[4 * q + 2],
                                         rr.w + v[4 * q + 3]);
                  reinterpret_cast<float4*>(o)[q] = w;
                }
              } else {
                for (int j = 0; j < 32 && nl0 + c + j < nlim; ++j) o[j] = r[j] + v[j];
              }
            } else {  // EPI_F32
              float* o = reinterpret_cast<float*>(p.out) + (size_t)m * p.ldo + n;
              if (full) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                  reinterpret_cast<float4*>(o)[q] =
                      make_float4(v[4 * q + 0], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
              } else {
                for (int j = 0; j < 32 && nl0 + c + j < nlim; ++j) o[j] = v[j];
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acce_bar(abuf));
      if (++abuf == 2) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
  }

  pdl_trigger();   // the next kernel may start its prologue while this CTA tears down
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ------------------------------------------------------------------ stream-K reduce + epilogue

enum DecEpi : int { DEC_BF16 = 0, DEC_RESID_F32 = 1, DEC_SWIGLU_BF16 = 2, DEC_F32 = 3 };

struct ReduceParams {
  int act_rows;         // tokens
  int n_out;            // output columns
  int num_kb;
  long long units;
  int grid;             // CTAs of the GEMM launch
  int max_pieces;
  int BN;               // token columns per partial piece
  int nseg;
  int seg_rows[3];
  int seg_tile0[4];
  int seg_col0[3];
  const float* partial;
  void* out;
  int ldo;
  const float* resid;
  int ldr;
  int ffn;              // DEC_SWIGLU: gate in segment 0, up in segment 1
};

// Sum of the stream-K pieces of weight row `wrow` (tile-local `r`) for token `t`.
// 32-bit arithmetic: the host guarantees units * grid < 2^32.
__device__ __forceinline__ float sk_sum(const ReduceParams& p, int wtile, int r, int t) {
  const unsigned U = (unsigned)p.units, G = (unsigned)p.grid, KB = (unsigned)p.num_kb;
  const unsigned x = (unsigned)wtile * KB;
  // largest CTA c with floor(U*c/G) <= x
  int c = (int)(((x + 1) * G + U - 1) / U) - 1;
  if (c < 0) c = 0;
  if (c > p.grid - 1) c = p.grid - 1;
  float s = 0.f;
  const unsigned xend = x + KB;
  for (; c < p.grid; ++c) {
    const unsigned start = U * (unsigned)c / G;
    if (start >= xend) break;
    const unsigned stop = U * (unsigned)(c + 1) / G;
    if (stop <= start) continue;
    const int slot = wtile - (int)(start / KB);
    s += p.partial[((size_t)c * p.max_pieces + slot) * (size_t)p.BN * 128 + (size_t)t * 128 + r];
  }
  return s;
}

__device__ __forceinline__ int seg_tile_of_row(const ReduceParams& p, int seg, int row_in_seg, int& r) {
  r = row_in_seg & 127;
  return p.seg_tile0[seg] + (row_in_seg >> 7);
}

template <int EPI>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const ReduceParams p) {
  pdl_wait();
  const int t = blockIdx.y;
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= p.act_rows || n >= p.n_out) return;
  if (EPI == DEC_SWIGLU_BF16) {
    int rg, ru;
    const int tg = seg_tile_of_row(p, 0, n, rg);
    const int tu = seg_tile_of_row(p, 1, n, ru);
    const float g = sk_sum(p, tg, rg, t);
    const float u = sk_sum(p, tu, ru, t);
    reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)t * p.ldo + n] = __float2bfloat16_rn(silu_f(g) * u);
    return;
  }
  int seg = 0;
  if (p.nseg > 1 && n >= p.seg_col0[1]) seg = 1;
  if (p.nseg > 2 && n >= p.seg_col0[2]) seg = 2;
  int r;
  const int wt = seg_tile_of_row(p, seg, n - p.seg_col0[seg], r);
  const float v = sk_sum(p, wt, r, t);
  if (EPI == DEC_BF16) {
    reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)t * p.ldo + n] = __float2bfloat16_rn(v);
  } else if (EPI == DEC_RESID_F32) {
    reinterpret_cast<float*>(p.out)[(size_t)t * p.ldo + n] = p.resid[(size_t)t * p.ldr + n] + v;
  } else {
    reinterpret_cast<float*>(p.out)[(size_t)t * p.ldo + n] = v;
  }
}

}  // namespace llama
