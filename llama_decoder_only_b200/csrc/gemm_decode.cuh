// Decode GEMMs (few token rows) with dynamically assigned chunks.
//
// Same operand roles as the stream-K form of gemm_tc_kernel: the weight fills
// the MMA's M = 128, the token rows are N = BN, and the (weight tile, k-block)
// units are laid out tile-major.  The units are cut into n_chunks equal
// chunks of consecutive units.  CTA i takes chunk i first -- known before the
// previous kernel ends, so its weight tiles are requested before the PDL wait
// -- and then grabs chunks grid, grid + 1, ... from a global counter, so SMs
// that stream faster take more chunks and all finish together (with an equal
// static split the slowest SM sets the kernel's time).
//
// A chunk covers one or two weight tiles; each part ("piece") of it is
// summed in TMEM.  A piece that covers a whole tile applies the epilogue at
// once.  Otherwise it writes its fp32 partial to its own slot and adds its
// k-block count to the tile's counter; the piece that brings the count to the
// tile's total adds all the tile's partials in chunk order (fixed, so the
// result does not depend on which piece finished last), applies the epilogue
// and re-arms the counter.  No CTA waits for another.
//
// Roles (320 threads): warp 0 producer (chunk grabs + TMA), warp 1 MMA
// issuer, warps 2-9 epilogue.  The producer hands each chunk id to the other
// two roles through a small ring in shared memory.
#pragma once

#include "gemm_tc.cuh"

namespace llama {

constexpr int DYN_QUEUE = 8;          // chunk-id ring between the producer and the other roles
constexpr int DYN_MAX_TILES = 512;    // tile counters in the workspace header

// A piece of chunk c: weight tile `tile`, k-blocks [kb0, kb1), index within the chunk.
struct DynPiece {
  int tile, kb0, kb1, idx;
};

// Pieces of chunk c (one or two): calls f(piece) in order.
template <typename F>
__device__ __forceinline__ void for_each_piece(const GemmParams& p, int c, F&& f) {
  const long long u0 = (long long)c * p.chunk_units;
  const long long u1 = min(p.units, u0 + p.chunk_units);
  const int t0 = (int)(u0 / p.num_kb);
  long long u = u0;
  int idx = 0;
  while (u < u1) {
    const int t = (int)(u / p.num_kb);
    const long long tend = min(u1, (long long)(t + 1) * p.num_kb);
    f(DynPiece{t, (int)(u - (long long)t * p.num_kb), (int)(tend - (long long)t * p.num_kb), t - t0});
    u = tend;
    ++idx;
  }
  (void)idx;
}

// Output column of weight-tile row `row` and whether it exists.
template <int EPI>
__device__ __forceinline__ void dyn_out_col(const GemmParams& p, int tile, int row, int& n, bool& n_ok) {
  if (EPI == EPI_SWIGLU_BF16) {
    n = tile * 64 + (row & 63);
    n_ok = n < p.seg_rows[0];
  } else {
    const int seg = seg_of_tile(p, tile);
    const int r_in_seg = (tile - p.seg_tile0[seg]) * 128 + row;
    n_ok = r_in_seg < p.seg_rows[seg];
    n = p.seg_col0[seg] + r_in_seg;
  }
}

// Apply the epilogue to 16 token columns [c, c + 16) of output column n.
template <int EPI, typename Sync>
__device__ __forceinline__ void dyn_apply16(const GemmParams& p, int n, bool n_ok, int c, bool active,
                                            const float (&v)[16], int row, float* xch, Sync& epi_sync) {
  if (EPI == EPI_SWIGLU_BF16) {
    // up values (lanes 64..127) go through shared memory to the gate lanes
    if (active && row >= 64) {
#pragma unroll
      for (int j = 0; j < 16; ++j) xch[j * 64 + row - 64] = v[j];
    }
    epi_sync();
    if (active && row < 64 && n_ok) {
      __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (c + j < p.act_rows) o[(size_t)(c + j) * p.ldo + n] = __float2bfloat16_rn(silu_f(v[j]) * xch[j * 64 + row]);
    }
    epi_sync();
  } else if (active && n_ok) {
    const int nj = p.act_rows - c < 16 ? p.act_rows - c : 16;
    if (EPI == EPI_RESID_F32) {
      // all residual loads first (out may alias resid: same element, same thread)
      float r[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) r[j] = j < nj ? p.resid[(size_t)(c + j) * p.ldr + n] : 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < nj) reinterpret_cast<float*>(p.out)[(size_t)(c + j) * p.ldo + n] = r[j] + v[j];
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j >= nj) break;
        const size_t o_idx = (size_t)(c + j) * p.ldo + n;
        if (EPI == EPI_BF16)
          reinterpret_cast<__nv_bfloat16*>(p.out)[o_idx] = __float2bfloat16_rn(v[j]);
        else
          reinterpret_cast<float*>(p.out)[o_idx] = v[j];
      }
    }
  }
}

template <int BN, int EPI, int KS>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_dyn_kernel(const __grid_constant__ CUtensorMap tmAct, const __grid_constant__ CUtensorMap tmW0,
                    const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2,
                    const GemmParams p) {
  using C = GemmCfg<BN, false, KS>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  float* xch_base = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES + 512);
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ int id_q[DYN_QUEUE];
  __shared__ int last_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  const uint32_t epi_bar = bar0 + 8u * (2 * STAGES + 5);
  auto idfull = [&](int q) { return bar0 + 8u * (2 * STAGES + 6 + q); };
  auto idempty = [&](int q) { return bar0 + 8u * (2 * STAGES + 6 + DYN_QUEUE + q); };
  static_assert(8 * (2 * STAGES + 6 + 2 * DYN_QUEUE) <= 512, "barrier area");

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
    mbar_init(epi_bar, 32 * GEMM_EPI_WARPS);
    for (int q = 0; q < DYN_QUEUE; ++q) {
      mbar_init(idfull(q), 1);
      mbar_init(idempty(q), 2);   // the MMA lane and the epilogue leader
    }
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmAct);
    tma_prefetch_desc(&tmW0);
    if (p.nseg > 1 || EPI == EPI_SWIGLU_BF16) tma_prefetch_desc(&tmW1);
    if (p.nseg > 2) tma_prefetch_desc(&tmW2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.early_trigger) pdl_trigger();
  if (warp != 0) pdl_wait();
  const uint32_t tmem_base = tmem_base_sh;
  WaitCtx wc{&abort_sh, p.status, p.limit_ns, 10};

  if (warp == 0) {
    // ------------------------------------------------------------ producer: chunk grabs + TMA
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int filled_parity[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) filled_parity[s] = -1;
      auto load_weight = [&](uint32_t sa, uint32_t bar, int wtile, int kb) {
#pragma unroll
        for (int i = 0; i < KS; ++i) {
          const int x = (kb * KS + i) * 64;
          const uint32_t dst = sa + i * C::A_SUB;
          if (EPI == EPI_SWIGLU_BF16) {
            tma_load_2d(dst, &tmW0, bar, x, wtile * 64);
            tma_load_2d(dst + 64 * 128, &tmW1, bar, x, wtile * 64);
          } else {
            const int seg = seg_of_tile(p, wtile);
            const CUtensorMap* wm = seg == 0 ? &tmW0 : (seg == 1 ? &tmW1 : &tmW2);
            tma_load_2d(dst, wm, bar, x, (wtile - p.seg_tile0[seg]) * 128);
          }
        }
      };
      auto load_act = [&](uint32_t sb, uint32_t bar, int kb) {
#pragma unroll
        for (int i = 0; i < KS; ++i) tma_load_2d(sb + i * C::B_SUB, &tmAct, bar, (kb * KS + i) * 64, 0);
      };
      // chunk blockIdx.x: its first stages' weights before the PDL wait
      int pre_kb[STAGES];
      int pre = 0;
      for_each_piece(p, blockIdx.x, [&](const DynPiece& pc) {
        for (int kb = pc.kb0; kb < pc.kb1 && pre < STAGES; ++kb) {
          mbar_arrive_expect_tx(full_bar(pre), C::STAGE_BYTES);
          load_weight(smem_u32(smem + pre * C::STAGE_BYTES), full_bar(pre), pc.tile, kb);
          pre_kb[pre++] = kb;
        }
      });
      pdl_wait();
      for (int s = 0; s < pre; ++s) {
        load_act(smem_u32(smem + s * C::STAGE_BYTES) + C::A_BYTES, full_bar(s), pre_kb[s]);
        filled_parity[s] = 0;
      }
      stage = pre % STAGES;
      phase = pre == STAGES ? 1u : 0u;
      int skip = pre;
      int c = blockIdx.x;
      bool ok = true;
      for (int qi = 0; ok; ++qi) {
        const int q = qi % DYN_QUEUE;
        if (!mbar_wait(idempty(q), ((qi / DYN_QUEUE) & 1) ^ 1u, wc, 20)) break;
        id_q[q] = c;
        mbar_arrive(idfull(q));   // release: the id is visible to the waiters
        if (c >= p.n_chunks) break;
        for_each_piece(p, c, [&](const DynPiece& pc) {
          for (int kb = pc.kb0; kb < pc.kb1 && ok; ++kb) {
            if (skip > 0) {
              --skip;
              continue;
            }
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc, 1)) {
              ok = false;
              break;
            }
            const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
            mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
            load_weight(sa, full_bar(stage), pc.tile, kb);
            load_act(sa + C::A_BYTES, full_bar(stage), kb);
            filled_parity[stage] = (int)phase;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        });
        c = (int)gridDim.x + (int)atomicAdd(p.dyn_ctr, 1u);
      }
      // every CTA has grabbed its last chunk once the count reaches the grid: the
      // last one re-arms the counters for the next launch
      __threadfence();
      if (atomicAdd(p.dyn_ctr + 1, 1u) == gridDim.x - 1) {
        atomicExch(p.dyn_ctr, 0u);
        atomicExch(p.dyn_ctr + 1, 0u);
      }
      for (int s = 0; s < STAGES; ++s)
        if (filled_parity[s] >= 0) mbar_wait(full_bar(s), (uint32_t)filled_parity[s], wc, 9, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, 0, 0);
      int stage = 0, abuf = 0;
      uint32_t phase = 0, aphase = 0;
      bool issued = false, ok = true;
      for (int qi = 0; ok; ++qi) {
        const int q = qi % DYN_QUEUE;
        if (!mbar_wait(idfull(q), (qi / DYN_QUEUE) & 1, wc, 21)) break;
        const int c = id_q[q];
        mbar_arrive(idempty(q));
        if (c >= p.n_chunks) break;
        for_each_piece(p, c, [&](const DynPiece& pc) {
          if (!ok) return;
          if (!mbar_wait(acce_bar(abuf), aphase ^ 1u, wc, 2)) {
            ok = false;
            return;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * BN);
          for (int kb = pc.kb0; kb < pc.kb1; ++kb) {
            if (!mbar_wait(full_bar(stage), phase, wc, 3)) {
              ok = false;
              return;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
            const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
            for (int i = 0; i < KS; ++i)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_bf16(d_tmem, smem_desc_sw128(sa + i * C::A_SUB + k * 32, 16, 1024),
                          smem_desc_sw128(sb + i * C::B_SUB + k * 32, 16, 1024), IDESC,
                          (kb > pc.kb0 || i > 0 || k > 0) ? 1u : 0u);
            issued = true;
            umma_commit(empty_bar(stage));
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          umma_commit(accf_bar(abuf));
          if (++abuf == 2) {
            abuf = 0;
            aphase ^= 1u;
          }
        });
      }
      if (issued) {
        umma_commit(drain_bar);
        mbar_wait(drain_bar, 0, wc, 8, false);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;   // TMEM lane == weight row of the tile
    const bool leader = threadIdx.x == 64;
    float* xch = xch_base + half * (64 * 16);
    uint32_t epi_phase = 0;
    auto epi_sync = [&]() {
      mbar_arrive(epi_bar);
      mbar_wait(epi_bar, epi_phase, wc, 7);
      epi_phase ^= 1u;
    };
    int abuf = 0;
    uint32_t aphase = 0;
    bool ok = true;
    constexpr size_t SLOT = (size_t)128 * BN;   // floats per partial slot
    for (int qi = 0; ok; ++qi) {
      const int q = qi % DYN_QUEUE;
      if (!__all_sync(0xffffffffu, mbar_wait(idfull(q), (qi / DYN_QUEUE) & 1, wc, 22))) break;
      const int c = id_q[q];
      epi_sync();   // every epilogue thread has read the id
      if (leader) mbar_arrive(idempty(q));
      if (c >= p.n_chunks) break;
      for_each_piece(p, c, [&](const DynPiece& pc) {
        if (!ok) return;
        if (!__all_sync(0xffffffffu, mbar_wait(accf_bar(abuf), aphase, wc, 4))) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(abuf * BN);
        int n;
        bool n_ok;
        dyn_out_col<EPI>(p, pc.tile, row, n, n_ok);
        const bool whole = pc.kb0 == 0 && pc.kb1 == p.num_kb;
        bool last = whole;
        if (!whole) {
          // publish this piece, then count its k-blocks on the tile
          float* dst = p.partial + ((size_t)(2 * c + pc.idx) * 128 + row) * BN;
#pragma unroll 1
          for (int col = half * 16; col < BN; col += 32) {
            float v[16];
            tmem_ld16(tbase + col, v);
            tmem_ld_wait();
            float4* d4 = reinterpret_cast<float4*>(dst + col);
#pragma unroll
            for (int k = 0; k < 4; ++k) d4[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          }
          epi_sync();   // every thread's stores precede the leader's release
          if (leader) {
            unsigned old;
            asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;"
                         : "=r"(old)
                         : "l"(p.tile_ctr + pc.tile), "r"((unsigned)(pc.kb1 - pc.kb0))
                         : "memory");
            last_sh = (old + (unsigned)(pc.kb1 - pc.kb0) == (unsigned)p.num_kb) ? 1 : 0;
          }
          epi_sync();
          last = last_sh != 0;
        }
        if (last) {
          // chunks that hold a piece of this tile, in order
          const int c_lo = (int)(((long long)pc.tile * p.num_kb) / p.chunk_units);
          const int c_hi = (int)(((long long)(pc.tile + 1) * p.num_kb - 1) / p.chunk_units);
#pragma unroll 1
          for (int col0 = 0; col0 < BN; col0 += 32) {
            const int col = col0 + half * 16;
            const bool active = col < BN;
            float v[16];
            if (active) {
              if (whole) {
                tmem_ld16(tbase + col, v);
                tmem_ld_wait();
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.f;
#pragma unroll 1
                for (int cc = c_lo; cc <= c_hi; ++cc) {
                  const int pidx = pc.tile - (int)(((long long)cc * p.chunk_units) / p.num_kb);
                  const float4* src =
                      reinterpret_cast<const float4*>(p.partial + ((size_t)(2 * cc + pidx) * 128 + row) * BN + col);
                  float4 a[4];
#pragma unroll
                  for (int k = 0; k < 4; ++k) a[k] = __ldcg(src + k);
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    v[4 * k + 0] += a[k].x;
                    v[4 * k + 1] += a[k].y;
                    v[4 * k + 2] += a[k].z;
                    v[4 * k + 3] += a[k].w;
                  }
                }
              }
            }
            dyn_apply16<EPI>(p, n, n_ok, col, active, v, row, xch, epi_sync);
          }
          // the tile is done: re-arm its counter for the next launch
          if (!whole && leader) asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p.tile_ctr + pc.tile), "r"(0u)
                                             : "memory");
        }
        (void)SLOT;
        tc_fence_before();
        mbar_arrive(acce_bar(abuf));
        if (++abuf == 2) {
          abuf = 0;
          aphase ^= 1u;
        }
      });
    }
  }

  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace llama
