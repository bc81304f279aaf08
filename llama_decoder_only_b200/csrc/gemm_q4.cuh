// Decode GEMMs with 4-bit group-64 weights ([MLX-13B] "LLaMA 2 的结构分析":
// every projection is a QuantizedLinear; "模型配置": quantization group_size 64,
// bits 4).  Reading of the format: per weight row and group of 64 inputs a
// scale s and an offset b, and per weight an unsigned code q in 0..15 with
// w = s * q + b; eight codes per 32-bit word, code k of the word in bits
// 4k .. 4k+3.
//
// The same swapped stream-K schedule as the bf16 decode GEMM (gemm_tc.cuh):
// the weight fills the MMA's M = 128, the few token rows are N = BN, the
// (weight tile, 64-wide k-block) units are split evenly over the CTAs and the
// CTA that ends a tile adds the others' pieces and applies the epilogue
// (streamk_epilogue).  What changes is the main loop -- a k-block of a
// weight tile is four quantisation groups:
//   warp 0       TMA producer: per unit of 4 groups (256 inputs), the packed
//                codes (128 rows x 128 contiguous bytes), the groups' scales
//                and offsets, and the activation tiles; the weight parts are
//                issued before the PDL wait (they do not depend on the
//                previous kernel), the activations after it;
//   warps 10-17  dequantisers: thread (row r, half h) owns groups h and h + 2
//                of weight row r; it turns 64 codes into bf16 w = fma(q, s, b)
//                (bf16x2 FMA, one rounding of the exact value) and writes them
//                into a 128-byte-swizzled K-major A tile per group, the layout
//                the MMA reads;
//   warp 1       MMA issuer: 4 x tcgen05.mma (M 128, N BN, K 16) per group
//                from the dequantised tile and the group's activation tile;
//   warps 2-9    stream-K epilogue.
// HBM moves 32 B of codes + 4 B of scale/offset per 64 weights: 0.5625 B per
// weight against 2 B in bf16.
#pragma once

#include "gemm_tc.cuh"

namespace llama {

constexpr int Q4_CONV_WARPS = 8;
constexpr int Q4_THREADS = GEMM_THREADS + 32 * Q4_CONV_WARPS;   // 576
constexpr int Q4_CONV_WARP0 = GEMM_THREADS / 32;                // 10
constexpr int Q4_KG = 4;                                        // quantisation groups (64 inputs) per unit

// One unit = one weight tile (128 rows) x Q4_KG groups: a stage reads 128
// contiguous bytes of codes of every row.
template <int BN>
struct Q4Cfg {
  static constexpr int ACT_SUB = BN * 64 * 2;                   // activation sub-tile of one group, swizzled
  static constexpr int ACT_BYTES = Q4_KG * ACT_SUB;
  static constexpr int CODE_BYTES = 128 * 32 * Q4_KG;           // 128 rows x 8 words per group
  static constexpr int SO_BYTES = 128 * 2 * Q4_KG;              // bf16 scales (or offsets): [half][group][64]
  static constexpr int STAGE_RAW = ACT_BYTES + CODE_BYTES + 2 * SO_BYTES;
  static constexpr int STAGE = (STAGE_RAW + 1023) / 1024 * 1024;
  static constexpr int A_BYTES = 128 * 128;                     // dequantised tile of one group
  static constexpr int LS_RAW = (120 * 1024) / STAGE;
  static constexpr int LSTAGES = LS_RAW < 2 ? 2 : (LS_RAW > 4 ? 4 : LS_RAW);
  static constexpr int AS_RAW = (204 * 1024 - LSTAGES * STAGE) / A_BYTES;
  static constexpr int ASTAGES = AS_RAW > 8 ? 8 : AS_RAW;
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128 : 256;
  static constexpr int EXCH_BYTES = 2 * 64 * 16 * 4;
  static constexpr int SMEM_BYTES = 1024 + LSTAGES * STAGE + ASTAGES * A_BYTES + 512 + EXCH_BYTES;
  static_assert(ASTAGES >= 2, "dequantised tile ring too small");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Tensor maps of one weight segment: codes uint32 [rows][K/8] (box 32 words
// x 64 rows), scales and offsets bf16 [K/64][rows] (box 64 rows x 4 groups).
struct Q4Maps {
  CUtensorMap codes[3], scales[3], offsets[3];
};

// 8 words (64 codes) of one row -> 64 bf16 weights s*q + b into row r of a
// 128-byte-swizzled K-major tile.
__device__ __forceinline__ void q4_dequant_row(const uint32_t* words, __nv_bfloat16 s, __nv_bfloat16 b,
                                               uint8_t* a_tile, int r) {
  const __nv_bfloat162 s2 = __bfloat162bfloat162(s), b2 = __bfloat162bfloat162(b);
  const __nv_bfloat162 c128 = __float2bfloat162_rn(128.0f);
  const uint4 w03 = *reinterpret_cast<const uint4*>(words);
  const uint4 w47 = *reinterpret_cast<const uint4*>(words + 4);
  const uint32_t wv[8] = {w03.x, w03.y, w03.z, w03.w, w47.x, w47.y, w47.z, w47.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t w = wv[j];
    // bytes (q0, q2, q4, q6) and (q1, q3, q5, q7), then interleaved: (q0..q3), (q4..q7)
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    const uint32_t t03 = __byte_perm(lo, hi, 0x5140), t47 = __byte_perm(lo, hi, 0x7362);
    // each code under the bf16 exponent byte of 128: the pairs (128 + q_2i, 128 + q_2i+1), exact
    const uint32_t e[4] = {__byte_perm(t03, 0x43434343u, 0x4140), __byte_perm(t03, 0x43434343u, 0x4342),
                           __byte_perm(t47, 0x43434343u, 0x4140), __byte_perm(t47, 0x43434343u, 0x4342)};
    uint32_t d[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 q = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&e[i]), c128);   // exact
      __nv_bfloat162 v = __hfma2(q, s2, b2);                                               // one rounding
      d[i] = *reinterpret_cast<uint32_t*>(&v);
    }
    *reinterpret_cast<uint4*>(a_tile + r * 128 + ((j ^ (r & 7)) << 4)) = make_uint4(d[0], d[1], d[2], d[3]);
  }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(Q4_THREADS, 1)
    gemm_q4_kernel(const __grid_constant__ CUtensorMap tmAct, const __grid_constant__ Q4Maps maps,
                   const GemmParams p) {
  using C = Q4Cfg<BN>;
  constexpr int LS = C::LSTAGES, AS = C::ASTAGES, KG = Q4_KG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_ring = smem + LS * C::STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(a_ring + AS * C::A_BYTES);
  float* xch_base = reinterpret_cast<float*>(a_ring + AS * C::A_BYTES + 512);
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float red_sh[GEMM_EPI_WARPS][16];   // fused RMSNorm: per-warp sums
  __shared__ float rstd_sh[128];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  // wfull: codes + scales + offsets of a unit landed; xfull: its activations
  // landed; lempty: the unit's MMAs are done; afull / aempty: one dequantised
  // group tile of the ring (tile t = unit * KG + group)
  auto wfull = [&](int s) { return bar0 + 8u * s; };
  auto xfull = [&](int s) { return bar0 + 8u * (LS + s); };
  auto lempty = [&](int s) { return bar0 + 8u * (2 * LS + s); };
  auto afull = [&](int a) { return bar0 + 8u * (3 * LS + a); };
  auto aempty = [&](int a) { return bar0 + 8u * (3 * LS + AS + a); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (3 * LS + 2 * AS + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (3 * LS + 2 * AS + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (3 * LS + 2 * AS + 4);
  const uint32_t epi_bar = bar0 + 8u * (3 * LS + 2 * AS + 5);
  static_assert(8 * (3 * LS + 2 * AS + 6) <= 512, "barrier area");

  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < LS; ++s) {
      mbar_init(wfull(s), 1);
      mbar_init(xfull(s), 1);
      mbar_init(lempty(s), 1);
    }
    for (int a = 0; a < AS; ++a) {
      mbar_init(afull(a), Q4_CONV_WARPS / 2);   // the four warps that own a group's rows
      mbar_init(aempty(a), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 32 * GEMM_EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    mbar_init(epi_bar, 32 * GEMM_EPI_WARPS);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmAct);
    for (int s = 0; s < p.nseg; ++s) {
      tma_prefetch_desc(&maps.codes[s]);
      tma_prefetch_desc(&maps.scales[s]);
      tma_prefetch_desc(&maps.offsets[s]);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.early_trigger) pdl_trigger();
  const uint32_t tmem_base = tmem_base_sh;
  WaitCtx wc{&abort_sh, p.status, p.limit_ns, 5};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // weight part of unit (wtile, kb) into stage s (no dependence on the previous kernel)
      auto load_weight = [&](int s, int wtile, int kb) {
        uint8_t* st = smem + s * C::STAGE;
        const uint32_t codes = smem_u32(st + C::ACT_BYTES);
        const uint32_t scl = codes + C::CODE_BYTES;
        const uint32_t off = scl + C::SO_BYTES;
        mbar_arrive_expect_tx(wfull(s), C::CODE_BYTES + 2 * C::SO_BYTES);
        for (int h = 0; h < 2; ++h) {
          int seg, r0;
          if (EPI == EPI_SWIGLU_BF16) {   // 64 gate rows, then the matching 64 up rows
            seg = h;
            r0 = wtile * 64;
          } else {
            seg = seg_of_tile(p, wtile);
            r0 = (wtile - p.seg_tile0[seg]) * 128 + 64 * h;
          }
          tma_load_2d(codes + h * (C::CODE_BYTES / 2), &maps.codes[seg], wfull(s), kb * 8 * KG, r0);
          tma_load_2d(scl + h * (C::SO_BYTES / 2), &maps.scales[seg], wfull(s), r0, kb * KG);
          tma_load_2d(off + h * (C::SO_BYTES / 2), &maps.offsets[seg], wfull(s), r0, kb * KG);
        }
      };
      auto load_act = [&](int s, int kb) {
        const uint32_t st = smem_u32(smem + s * C::STAGE);
        mbar_arrive_expect_tx(xfull(s), C::ACT_BYTES);
#pragma unroll
        for (int g = 0; g < KG; ++g) tma_load_2d(st + g * C::ACT_SUB, &tmAct, xfull(s), (kb * KG + g) * 64, 0);
      };
      int wfilled[LS], xfilled[LS];
#pragma unroll
      for (int s = 0; s < LS; ++s) wfilled[s] = xfilled[s] = -1;
      // the first LS units' weights before the PDL wait
      int pre_kb[LS];
      int pre = 0;
      {
        GemmIter it;
        it.init(p, true);
        GemmItem item;
        while (pre < LS && it.next(item))
          for (int kb = item.kb0; kb < item.kb1 && pre < LS; ++kb) {
            load_weight(pre, item.tile, kb);
            wfilled[pre] = 0;
            pre_kb[pre++] = kb;
          }
      }
      pdl_wait();
      for (int s = 0; s < pre; ++s) {
        load_act(s, pre_kb[s]);
        xfilled[s] = 0;
      }
      GemmIter it;
      it.init(p, true);
      GemmItem item;
      long long u = 0;
      bool ok = true;
      while (ok && it.next(item)) {
        for (int kb = item.kb0; kb < item.kb1; ++kb, ++u) {
          if (u < pre) continue;
          const int s = (int)(u % LS);
          const uint32_t ph = (uint32_t)((u / LS) & 1);
          if (!mbar_wait(lempty(s), ph ^ 1u, wc, 1)) {
            ok = false;
            break;
          }
          load_weight(s, item.tile, kb);
          load_act(s, kb);
          wfilled[s] = xfilled[s] = (int)ph;
        }
      }
      for (int s = 0; s < LS; ++s) {
        if (wfilled[s] >= 0) mbar_wait(wfull(s), (uint32_t)wfilled[s], wc, 9, false);
        if (xfilled[s] >= 0) mbar_wait(xfull(s), (uint32_t)xfilled[s], wc, 9, false);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, 0, 0);
      int abuf = 0;
      uint32_t aphase = 0;
      bool issued = false, ok = true;
      long long u = 0;
      GemmIter it;
      it.init(p, true);
      GemmItem item;
      while (ok && it.next(item)) {
        if (!mbar_wait(acce_bar(abuf), aphase ^ 1u, wc, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * BN);
        for (int kb = item.kb0; kb < item.kb1 && ok; ++kb, ++u) {
          const int s = (int)(u % LS);
          if (!mbar_wait(xfull(s), (uint32_t)((u / LS) & 1), wc, 3)) {
            ok = false;
            break;
          }
          const uint32_t sb = smem_u32(smem + s * C::STAGE);
          for (int g = 0; g < KG; ++g) {
            const long long t = u * KG + g;
            const int a = (int)(t % AS);
            if (!mbar_wait(afull(a), (uint32_t)((t / AS) & 1), wc, 3)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(a_ring + a * C::A_BYTES);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16(d_tmem, smem_desc_sw128(sa + k * 32, 16, 1024),
                        smem_desc_sw128(sb + g * C::ACT_SUB + k * 32, 16, 1024), IDESC,
                        (kb > item.kb0 || g > 0 || k > 0) ? 1u : 0u);
            issued = true;
            umma_commit(aempty(a));
          }
          if (!ok) break;
          umma_commit(lempty(s));
        }
        if (!ok) break;
        umma_commit(accf_bar(abuf));
        if (++abuf == 2) {
          abuf = 0;
          aphase ^= 1u;
        }
      }
      if (issued) {
        umma_commit(drain_bar);
        mbar_wait(drain_bar, 0, wc, 8, false);
      }
    }
  } else if (warp >= Q4_CONV_WARP0) {
    // ------------------------------------------------------------ dequantisers
    // thread (row r, half h): groups h and h + 2 of every unit
    const int ct = (warp - Q4_CONV_WARP0) * 32 + lane;
    const int r = ct & 127, h = ct >> 7;
    long long u = 0;
    bool ok = true;
    GemmIter it;
    it.init(p, true);
    GemmItem item;
    while (ok && it.next(item)) {
      for (int kb = item.kb0; kb < item.kb1; ++kb, ++u) {
        const int s = (int)(u % LS);
        if (!__all_sync(0xffffffffu, mbar_wait(wfull(s), (uint32_t)((u / LS) & 1), wc, 10))) {
          ok = false;
          break;
        }
        const uint8_t* st = smem + s * C::STAGE + C::ACT_BYTES;
        const uint32_t* words = reinterpret_cast<const uint32_t*>(st) + r * (8 * KG);
        const __nv_bfloat16* scl = reinterpret_cast<const __nv_bfloat16*>(st + C::CODE_BYTES);
        const __nv_bfloat16* ofs = reinterpret_cast<const __nv_bfloat16*>(st + C::CODE_BYTES + C::SO_BYTES);
        const int so = (r >> 6) * (64 * KG) + (r & 63);   // [half][group][64]
        for (int g = h; g < KG; g += 2) {
          const long long t = u * KG + g;
          const int a = (int)(t % AS);
          if (!__all_sync(0xffffffffu, mbar_wait(aempty(a), (uint32_t)(((t / AS) & 1) ^ 1), wc, 11))) {
            ok = false;
            break;
          }
          q4_dequant_row(words + 8 * g, scl[so + 64 * g], ofs[so + 64 * g], a_ring + a * C::A_BYTES, r);
          fence_proxy_async_smem();   // generic-proxy stores -> visible to the tensor core
          __syncwarp();
          if (lane == 0) mbar_arrive(afull(a));
        }
        if (!ok) break;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    uint32_t epi_phase = 0;
    auto epi_sync = [&]() {
      mbar_arrive(epi_bar);
      mbar_wait(epi_bar, epi_phase, wc, 7);
      epi_phase ^= 1u;
    };
    int abuf = 0;
    uint32_t aphase = 0;
    GemmIter it;
    it.init(p, true);
    GemmItem item;
    pdl_wait();   // residuals and the flag words are written by earlier kernels
    while (it.next(item)) {
      if (!__all_sync(0xffffffffu, mbar_wait(accf_bar(abuf), aphase, wc, 4))) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(abuf * BN);
      streamk_epilogue<BN, EPI>(p, item, tbase, row, half, xch_base + half * (64 * 16), threadIdx.x == 64,
                                &abort_sh, epi_sync, red_sh);
      tc_fence_before();
      mbar_arrive(acce_bar(abuf));
      if (++abuf == 2) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
    if constexpr (EPI == EPI_RESID_F32)
      if (p.norm_g != nullptr) fused_rmsnorm<BN>(p, threadIdx.x == 64, &abort_sh, epi_sync, rstd_sh);
  }

  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace llama
