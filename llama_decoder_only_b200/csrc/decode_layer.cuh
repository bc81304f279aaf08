// One decode step of a whole block in one persistent kernel (batch <= 16).
//
// At a handful of token rows a decode block is a stream of weight bytes
// (every projection is GEMV-shaped) with small dependent steps in between:
// RMSNorm ([MLX-13B] 4. RMSNorm), the Q/K/V projection, RoPE + KV append and
// attention over the cache ([MLX-13B] 2. 注意力机制, 3. RoPE; [DeepDive]
// LLaMAAttention), o_proj + residual, RMSNorm, gate/up + SiLU·mul, down +
// residual ([DeepDive] LLaMAMLP, LLaMADecoderLayer).  As separate kernels
// every step pays its start-up and its fix-up tail with HBM idle.  Here one
// CTA per SM runs all steps as phases separated by grid-wide barriers, and
// the TMA producer warp of every CTA keeps streaming: before each projection
// waits for its activation, the producer has already filled every free stage
// of its ring with that projection's weight tiles (weights do not depend on
// the step before).
//
// Roles (320 threads): warp 0 producer (TMA), warp 1 MMA issuer (tcgen05,
// swapped: weight rows fill M = 128, the token rows are N = 16, accumulator
// in TMEM), warps 2..9 workers: the stream-K epilogues of the projections
// (the same code as the stand-alone decode GEMM), the two RMSNorms, and the
// attention (two groups of four warps, one (sequence, KV head) each, with
// RoPE + KV append inside, one key split).
//
// Phases and grid barriers (one counter per barrier; barrier k completes when
// every CTA has arrived at it -- a single running count would let a CTA with
// no work in a phase arrive at the next barrier early and stand in for one
// still busy):
//   P0 RMSNorm-1: every CTA's share of each row's sum of squares    -> 0
//      then rstd of every row from the shares, its column slice of h -> 1
//   P1 QKV projection into qkv (raw)                                  -> 2
//   P2 RoPE + KV append + attention into att                          -> 3
//   P3 o_proj + residual into x_out (x_mid), per-tile sums of squares -> 4
//   P4 RMSNorm-2 (its column slice of h)                              -> 5
//   P5 gate/up + SiLU·mul into m                                      -> 6
//   P6 down + residual into x_out
// The producer waits for barrier 1 / 3 / 5 / 6 before the activation tiles of
// P1 / P3 / P5 / P6; the workers wait for 2 and 4 before P2 and P4.  Every
// wait is bounded (the workspace status word records a timeout).  All CTAs
// must be resident at once: the kernel is launched cooperatively with one
// CTA per SM.
#pragma once

#include <type_traits>

#include "attention.cuh"
#include "gemm_tc.cuh"

namespace llama {

constexpr int DL_BN = 16;   // token columns of the swapped MMA: batch <= 16
constexpr int DL_KS = 2;    // 64-wide k sub-blocks per stage
using DLCfg = GemmCfg<DL_BN, false, DL_KS>;

enum DlGemm : int { DL_QKV = 0, DL_O = 1, DL_GU = 2, DL_DOWN = 3 };

struct alignas(64) DecLayerParams {
  CUtensorMap act[4];     // activation (B operand) of each projection: h, att, h, m
  CUtensorMap w[4][3];    // weight maps: QKV (1 or 3 segments), o_proj, gate / up, down
  GemmParams g[4];        // stream-K parameters of each projection
  AttnDecodeParams attn;  // raw qkv, caches, T = cache length after the append, RoPE; out = att
  const float* x_in;      // [B, dim] block input
  float* x_out;           // [B, dim] x_mid after o_proj, the block output after down
  const float* attn_norm; // [dim]
  const float* ffn_norm;
  __nv_bfloat16* h;       // [B, dim] RMSNorm output (first RMSNorm-1, then RMSNorm-2)
  float* ssq;             // [o_proj tiles][16] per-tile sums of squares of x_mid rows
  float* slots;           // [CTAs][16] each CTA's share of the sums of squares of the x_in rows
  unsigned* bar;          // [8] grid barriers 0..6 at [0..6], CTAs done at [7]
  DevStatus* status;
  unsigned long long limit_ns;
  float eps;
  int dim, B;
  int l2_prefetch;        // 1: the producer prefetches upcoming weights and the cache into L2
};
static_assert(sizeof(DecLayerParams) <= 4096, "kernel parameters exceed 4 KB");

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// L2 prefetch of one box of a tensor map (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* m, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y)
               : "memory");
}
// L2 prefetch of a contiguous range (16-byte aligned address and size).
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes) : "memory");
}

// Bytes each L2 prefetch batch of the producer may bring in, over all CTAs: a
// few batches stay well inside the 126 MB L2.
constexpr long long kDlPrefetchBatch = 32ll << 20;

// Bounded wait until every CTA has arrived at a grid barrier (its counter
// reaches `target`).
__device__ __forceinline__ bool dl_grid_wait(const unsigned* bar, unsigned target, int* abort_sh, DevStatus* st,
                                             unsigned long long limit_ns, int detail) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
    if (v >= target) return true;
    if (*reinterpret_cast<volatile int*>(abort_sh)) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_sh = 1;
      record_error(st, LLAMA_ERR_DEVICE_TIMEOUT, 12, detail);
      return false;
    }
    __nanosleep(32);
  }
}

template <int HD, int G>
struct DecLayerSmem {
  static constexpr int RING = DLCfg::STAGES * DLCfg::STAGE_BYTES;
  static constexpr int BARS = 256;
  static constexpr int XCH = DLCfg::EXCH_BYTES;
  static constexpr int ATT = 2 * (int)sizeof(DecAttnSmem<HD, G>);
  static constexpr int BYTES = 1024 + RING + BARS + XCH + ATT;
};

template <int HD, int G>
// 320 threads at one CTA per SM: ptxas caps the kernel at 168 registers a
// thread (a 200-register build failed to launch).
__global__ void __launch_bounds__(GEMM_THREADS, 1) decode_layer_kernel(const __grid_constant__ DecLayerParams P) {
  using C = DLCfg;
  using S = DecLayerSmem<HD, G>;
  constexpr int STAGES = C::STAGES;
  constexpr int BN = DL_BN, KS = DL_KS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::RING);
  float* xch = reinterpret_cast<float*>(smem + S::RING + S::BARS);
  DecAttnSmem<HD, G>* ash = reinterpret_cast<DecAttnSmem<HD, G>*>(smem + S::RING + S::BARS + S::XCH);
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float red_sh[GEMM_EPI_WARPS][16];
  __shared__ float rstd_sh[16];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned nctas = gridDim.x;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  const uint32_t epi_bar = bar0 + 8u * (2 * STAGES + 5);

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
    fence_barrier_init();
  }
  if (warp == 0 && lane < 4) {
    tma_prefetch_desc(&P.act[lane]);
    for (int s = 0; s < 3; ++s) tma_prefetch_desc(&P.w[lane][s]);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();   // x_in and the cache come from earlier kernels
  const uint32_t tmem_base = tmem_base_sh;
  WaitCtx wc{&abort_sh, P.status, P.limit_ns, 12};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int filled_parity[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) filled_parity[s] = -1;
      bool ok = true;
      constexpr unsigned kBarrierBefore[4] = {1, 3, 5, 6};
      const long long budget = kDlPrefetchBatch / nctas;   // bytes per CTA and batch
      // L2 prefetch of this CTA's weight tiles of projection gj in the order it
      // will load them, after its first `skip` units, up to `budget` bytes
      auto prefetch_weights = [&](int gj, int skip) {
        const GemmParams& q = P.g[gj];
        GemmIter it;
        it.init(q, true);
        GemmItem item;
        int n = 0;
        long long bytes = 0;
        while (it.next(item)) {
          for (int kb = item.kb0; kb < item.kb1; ++kb) {
            if (n++ < skip) continue;
            if (bytes >= budget) return;
#pragma unroll
            for (int i = 0; i < KS; ++i) {
              const int x = (kb * KS + i) * 64;
              if (gj == DL_GU) {
                tma_prefetch_l2_2d(&P.w[gj][0], x, item.tile * 64);
                tma_prefetch_l2_2d(&P.w[gj][1], x, item.tile * 64);
              } else {
                const int seg = seg_of_tile(q, item.tile);
                tma_prefetch_l2_2d(&P.w[gj][seg], x, (item.tile - q.seg_tile0[seg]) * 128);
              }
            }
            bytes += C::A_BYTES;
          }
        }
      };
      // L2 prefetch of the cached keys and values [0, T-1) of this CTA's
      // attention units (the new token's row is appended during the step)
      auto prefetch_kv = [&]() {
        const AttnDecodeParams& a = P.attn;
        const long long row_bytes = (long long)HD * 2;
        const long long n_bytes = (long long)(a.T - 1) * row_bytes;
        const int units = P.B * a.nkv;
        long long bytes = 0;
        // the units of this CTA's two worker groups, round by round
        for (int u0 = (int)blockIdx.x * 2; u0 < units && bytes < budget; u0 += 2 * (int)nctas) {
          for (int u = u0; u < u0 + 2 && u < units; ++u) {
            const int b = u / a.nkv, g = u - b * a.nkv;
            const size_t off = ((size_t)b * a.nkv + g) * (size_t)a.cap * HD;
            for (long long o = 0; o < n_bytes; o += 32768) {
              const uint32_t len = (uint32_t)min(32768ll, n_bytes - o);
              bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(a.kc + off) + o, len);
              bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(a.vc + off) + o, len);
            }
            bytes += 2 * n_bytes;
          }
        }
      };
#pragma unroll 1
      for (int gi = 0; gi < 4 && ok; ++gi) {
        const GemmParams& p = P.g[gi];
        const CUtensorMap* wmaps = P.w[gi];
        auto load_weight = [&](uint32_t sa, uint32_t bar, int wtile, int kb) {
#pragma unroll
          for (int i = 0; i < KS; ++i) {
            const int x = (kb * KS + i) * 64;
            const uint32_t dst = sa + i * C::A_SUB;
            if (gi == DL_GU) {
              tma_load_2d(dst, &wmaps[0], bar, x, wtile * 64);
              tma_load_2d(dst + 64 * 128, &wmaps[1], bar, x, wtile * 64);
            } else {
              const int seg = seg_of_tile(p, wtile);
              tma_load_2d(dst, &wmaps[seg], bar, x, (wtile - p.seg_tile0[seg]) * 128);
            }
          }
        };
        auto load_act = [&](uint32_t sb, uint32_t bar, int kb) {
#pragma unroll
          for (int i = 0; i < KS; ++i) tma_load_2d(sb + i * C::B_SUB, &P.act[gi], bar, (kb * KS + i) * 64, 0);
        };
        // 1. weight tiles into every stage that frees up, before the activation exists
        int pre = 0, pre_stage[STAGES], pre_kb[STAGES];
        {
          GemmIter it;
          it.init(p, true);
          GemmItem item;
          while (ok && pre < STAGES && it.next(item)) {
            for (int kb = item.kb0; kb < item.kb1 && pre < STAGES; ++kb) {
              if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc, 1)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
              load_weight(smem_u32(smem + stage * C::STAGE_BYTES), full_bar(stage), item.tile, kb);
              filled_parity[stage] = (int)phase;
              pre_stage[pre] = stage;
              pre_kb[pre++] = kb;
              if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
              }
            }
          }
        }
        if (!ok) break;
        // keep HBM busy through the phases that stream no weights: the next
        // bytes this CTA will want go to L2 now (one projection ahead, and the
        // attention's keys and values during the QKV projection)
        if (!P.l2_prefetch) {
        } else if (gi == DL_QKV) {
          prefetch_weights(DL_QKV, STAGES);
          prefetch_kv();
          prefetch_weights(DL_O, STAGES);
        } else if (gi == DL_O) {
          prefetch_weights(DL_GU, STAGES);
        } else if (gi == DL_GU) {
          prefetch_weights(DL_DOWN, STAGES);
        }
        // 2. the activation of this projection is complete in every CTA
        if (!dl_grid_wait(P.bar + kBarrierBefore[gi], nctas, &abort_sh, P.status, P.limit_ns, gi)) break;
        fence_proxy_async_global();
        for (int i = 0; i < pre; ++i)
          load_act(smem_u32(smem + pre_stage[i] * C::STAGE_BYTES) + C::A_BYTES, full_bar(pre_stage[i]), pre_kb[i]);
        // 3. the rest of this CTA's units
        int skip = pre;
        GemmIter it;
        it.init(p, true);
        GemmItem item;
        while (ok && it.next(item)) {
          for (int kb = item.kb0; kb < item.kb1; ++kb) {
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
            load_weight(sa, full_bar(stage), item.tile, kb);
            load_act(sa + C::A_BYTES, full_bar(stage), kb);
            filled_parity[stage] = (int)phase;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      // drain: every issued fill lands before the CTA may exit
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
      bool issued = false, ok = true;
#pragma unroll 1
      for (int gi = 0; gi < 4 && ok; ++gi) {
        GemmIter it;
        it.init(P.g[gi], true);
        GemmItem item;
        while (ok && it.next(item)) {
          if (!mbar_wait(acce_bar(abuf), aphase ^ 1u, wc, 2)) {
            ok = false;
            break;
          }
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
            for (int i = 0; i < KS; ++i)
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t ad = smem_desc_sw128(sa + i * C::A_SUB + k * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(sb + i * C::B_SUB + k * 32, 16, 1024);
                umma_bf16(d_tmem, ad, bd, IDESC, (kb > item.kb0 || i > 0 || k > 0) ? 1u : 0u);
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
      }
      if (issued) {
        umma_commit(drain_bar);
        mbar_wait(drain_bar, 0, wc, 8, false);
      }
    }
  } else {
    // ------------------------------------------------------------ workers (warps 2..9)
    const int wid = threadIdx.x - 64;          // 0 .. 255
    const int ww = wid >> 5;                   // worker warp 0 .. 7
    const bool leader = wid == 0;
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may read
    const int half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    uint32_t epi_phase = 0;
    auto epi_sync = [&]() {
      mbar_arrive(epi_bar);
      mbar_wait(epi_bar, epi_phase, wc, 7);
      epi_phase ^= 1u;
    };
    // this CTA's writes of the phase are done: count it at grid barrier k
    auto arrive = [&](int k) {
      fence_proxy_async_global();   // readers of these writes include TMA loads
      epi_sync();
      if (leader) {
        __threadfence();
        asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(P.bar + k), "r"(1u) : "memory");
      }
    };
    auto grid_wait = [&](int k) {
      if (leader) dl_grid_wait(P.bar + k, nctas, &abort_sh, P.status, P.limit_ns, 10 + k);
      epi_sync();
      return *reinterpret_cast<volatile int*>(&abort_sh) == 0;
    };
    int abuf = 0;
    uint32_t aphase = 0;
    auto epilogues = [&](auto epi_tag, int gi) {
      constexpr int EPI = decltype(epi_tag)::value;
      GemmIter it;
      it.init(P.g[gi], true);
      GemmItem item;
      while (it.next(item)) {
        if (!__all_sync(0xffffffffu, mbar_wait(accf_bar(abuf), aphase, wc, 4))) break;
        tc_fence_after();
        const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(abuf * BN);
        streamk_epilogue<BN, EPI>(P.g[gi], item, tbase, row, half, xch + half * (64 * 16), leader, &abort_sh,
                                  epi_sync, red_sh);
        tc_fence_before();
        mbar_arrive(acce_bar(abuf));
        if (++abuf == 2) {
          abuf = 0;
          aphase ^= 1u;
        }
      }
    };
    const int dim = P.dim, B = P.B;
    const int n0 = (int)((long long)dim * blockIdx.x / nctas);
    const int n1 = (int)((long long)dim * (blockIdx.x + 1) / nctas);
    // h[:, n0:n1] = bf16(g * (x * rstd)), rstd of each row already in rstd_sh
    auto norm_slice = [&](const float* x, const float* gw) {
      const int w = n1 - n0;
      for (int i = wid; i < w * B; i += 32 * GEMM_EPI_WARPS) {
        const int j = i / w, n = n0 + i % w;
        P.h[(size_t)j * dim + n] = __float2bfloat16_rn(__ldg(gw + n) * (__ldcg(x + (size_t)j * dim + n) * rstd_sh[j]));
      }
    };

    // the new token's RoPE angles, the same for every unit of the attention
    // phase (one position per step), once per group
    dec_attn_angles<HD, G>(P.attn, 0, wid & 127, ash[wid >> 7]);
    // P0: RMSNorm-1.  Each CTA sums the squares of its own columns of every
    // row (16 threads a row), the shares meet at barrier 0, and every CTA adds
    // the shares in CTA order (the same rstd everywhere) for its column slice.
    {
      const int j = wid >> 4, r = wid & 15;
      float q = 0.f;
      if (j < B)
        for (int n = n0 + r; n < n1; n += 16) {
          const float v = __ldcg(P.x_in + (size_t)j * dim + n);
          q = fmaf(v, v, q);
        }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
      if (j < B && r == 0) P.slots[blockIdx.x * 16 + j] = q;
    }
    arrive(0);
    if (grid_wait(0)) {
      const int j = wid >> 4, r = wid & 15;
      float q = 0.f;
      if (j < B)
        for (int c = r; c < (int)nctas; c += 16) q += __ldcg(P.slots + c * 16 + j);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
      if (j < B && r == 0) rstd_sh[j] = rsqrtf(q / (float)dim + P.eps);
    }
    epi_sync();
    norm_slice(P.x_in, P.attn_norm);
    arrive(1);
    // P1: QKV projection (raw q, k, v)
    epilogues(std::integral_constant<int, EPI_BF16>{}, DL_QKV);
    arrive(2);
    // P2: RoPE + KV append + attention, one (sequence, KV head) per group of four warps
    if (grid_wait(2)) {
      const int grp = wid >> 7, tid = wid & 127;
      const int units = B * P.attn.nkv;
      DecAttnSmem<HD, G>& sh = ash[grp];
      auto group_sync = [grp] { asm volatile("bar.sync %0, 128;" ::"r"(1 + grp) : "memory"); };
      for (int u = (int)blockIdx.x * 2 + grp; u < units; u += 2 * (int)nctas) {
        const int b = u / P.attn.nkv, g = u - b * P.attn.nkv;
        attn_decode_body<HD, G, true>(P.attn, 0, g, b, tid, sh, group_sync);
        group_sync();   // the group's shared state is free for its next unit
      }
    }
    arrive(3);
    // P3: o_proj + residual -> x_mid, with each tile's sums of squares
    epilogues(std::integral_constant<int, EPI_RESID_F32>{}, DL_O);
    arrive(4);
    // P4: RMSNorm-2 from the tiles' sums of squares
    if (grid_wait(4)) {
      for (int j = ww; j < B; j += GEMM_EPI_WARPS) {
        float q = 0.f;
        for (int t = lane; t < P.g[DL_O].n_tiles; t += 32) q += __ldcg(P.ssq + (size_t)t * BN + j);
        q = warp_sum(q);
        if (lane == 0) rstd_sh[j] = rsqrtf(q / (float)dim + P.eps);
      }
      epi_sync();
      norm_slice(P.x_out, P.ffn_norm);
    }
    arrive(5);
    // P5: gate/up + SiLU·mul -> m
    epilogues(std::integral_constant<int, EPI_SWIGLU_BF16>{}, DL_GU);
    arrive(6);
    // P6: down + residual -> block output
    epilogues(std::integral_constant<int, EPI_RESID_F32>{}, DL_DOWN);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
  if (threadIdx.x == 0) {
    // the last CTA to finish re-arms the barrier words for the next launch
    // (every CTA has passed all its waits by the time it counts itself here)
    __threadfence();
    if (atomicAdd(P.bar + 7, 1u) == nctas - 1) {
      for (int k = 0; k < 8; ++k) atomicExch(P.bar + k, 0u);
    }
  }
}

}  // namespace llama
