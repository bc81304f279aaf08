// Causal grouped-query attention over the KV cache, bf16 operands.
//
//  * attn_prefill_kernel: flash attention on tcgen05 ([HandsOn] "Transformer
//    块的内部结构" names FlashAttention: tile Q/K/V through on-chip memory
//    instead of materialising the score matrix in HBM).  One CTA per
//    (256-query block, head, sequence) = two 128-row query tiles that share
//    every K/V tile (for GQA: two query heads of one KV group over 128 query
//    rows); K/V tiles of 128 keys arrive by TMA into a 4-slot ring;
//    S_t = Q_t K^T lands in TMEM, a softmax warpgroup per tile reads it with
//    tcgen05.ld, keeps the running max / sum in fp32 (online softmax), writes
//    P_t as bf16 back into TMEM over S_t (tcgen05.st), and the MMA warp
//    accumulates O_t += P_t V with P_t as the TMEM A operand; the two tiles
//    ping-pong so one tile's softmax overlaps the other tile's MMAs.  The running max is only moved (and
//    O rescaled) when it grows by more than 2^8, which is exact because the
//    final division uses the same stale maximum for numerator and sum.
//  * attn_prefill_k64_kernel (head_dim below 128): the same with 64-key
//    steps and two S buffers per query tile, so a tile's next S is computed
//    while its softmax runs.
//  * attn_decode_kernel (and attn_decode_mma_kernel for GQA groups >= 4):
//    one new query per sequence; the cache of each (sequence, KV head) is
//    split along the key axis over several CTAs; the query heads of a GQA
//    group share every K/V load; partial (max, sum, output) are merged with
//    the usual log-sum-exp rule by attn_decode_combine_kernel.
//    CUDA-core FMAs, 16-byte loads; bound by HBM bandwidth.
//
// Definition followed: softmax(q k^T / sqrt(hd)) v over keys j <= p
// ([MLX-13B] 2. 注意力机制 and 5. 因果掩码; [DeepDive] LLaMAAttention),
// query head h reads KV head h / (nh / nkv).
#pragma once

#include "common.cuh"
#include "ragged.cuh"
#include "small_kernels.cuh"

namespace llama {

constexpr float kLog2e = 1.4426950408889634f;

// ====================================================================== prefill

struct AttnPrefillParams {
  int L;         // new tokens per sequence
  int p0;        // position of token 0 (cache length before the call)
  int nh, nkv, hd;
  int n_qblocks; // query blocks per (head pair or head, sequence)
  // 1: a CTA takes two query heads of one KV group over the same 128 query
  // rows (GQA, group >= 2: every K/V tile serves both heads); 0: one head over
  // 256 query rows (two 128-row tiles)
  int head_pair;
  float scale_log2;   // log2(e) / sqrt(hd)
  __nv_bfloat16* out; // [B*L, nh*hd] (ragged: [sum of new tokens, nh*hd])
  DevStatus* status;
  unsigned long long limit_ns;
  // ragged batch: sequence b has tab->len[b] new tokens at packed rows
  // tab->start[b] .., positions tab->p0[b] ..; tmQ is then a 2-D map over the
  // packed rows.  nullptr: every sequence has L tokens at positions p0 ...
  const SeqTab* tab;
};

constexpr int ATT_REGION = 128 * 128;           // bytes of a [128 rows x 64 bf16] region
constexpr int ATT_TILE = 2 * ATT_REGION;        // one 128-row tile of a head (two 64-column regions)
constexpr int ATT_SLOTS = 4;                    // K/V ring: K_j, V_j, K_{j+1}, V_{j+1} in flight
constexpr int ATT_THREADS = 320;                // producer, MMA, 2 softmax warpgroups
constexpr int ATT_SMEM = 1024 + 2 * ATT_TILE    // Q0, Q1
                         + ATT_SLOTS * ATT_TILE  // K/V ring
                         + 256;

// 32 lanes x 16 consecutive 32-bit columns from registers (thread t -> lane
// quadrant*32 + t), the store form of tmem_ld16.
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  __syncwarp();
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two 128-row query tiles (t = 0, 1) of one head share every K/V tile.  The
// MMA warp interleaves S1_j, P0·V_j, S0_{j+1}, P1·V_j, so while one softmax
// warpgroup turns S_t into P_t the tensor core works on the other tile.
// One CTA per SM (shared memory).  __launch_bounds__ lets ptxas pick the
// register split; an explicit cap of 192 or 200 registers failed to launch
// ("too many resources") at 320 threads.
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnPrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                   // tile t at t * ATT_TILE
  uint8_t* sKV = sQ + 2 * ATT_TILE;                     // slot s at s * ATT_TILE
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + ATT_SLOTS * ATT_TILE);
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Causal work grows with the query block.  CTAs are dispatched x-fastest, so
  // with the block index in z every (head, sequence) starts its heaviest
  // (latest) block in the first wave and the light ones fill in behind.
  const int qb = p.n_qblocks - 1 - blockIdx.z;
  const int b = blockIdx.y;
  const bool hp = p.head_pair != 0;
  // query tile t: head h_t, rows q_row0 + qoff_t of the sequence
  const int h0 = hp ? 2 * blockIdx.x : blockIdx.x;
  const int g = h0 / (p.nh / p.nkv);             // both heads of a pair share it
  const int hd = p.hd;
  const int nreg = hd > 64 ? 2 : 1;             // 64-column regions per head row
  const int hd_pad = nreg * 64;
  const int q_row0 = qb * (hp ? 128 : 256);
  const int qoff1 = hp ? 0 : 128;                // rows of tile 1 after q_row0
  // this sequence's new tokens, their first position and first packed row
  int Ls = p.L, p0s = p.p0, row_base = b * p.L;
  if (p.tab != nullptr) {
    pdl_wait();   // the table is written by an earlier kernel
    Ls = p.tab->len[b];
    p0s = p.tab->p0[b];
    row_base = p.tab->start[b];
  }
  const bool q0_valid = q_row0 < Ls;
  const bool q1_valid = q_row0 + qoff1 < Ls;
  // kv tiles with any key visible to tile t (0 for an empty tile)
  const int last0 = min(Ls, q_row0 + 128) - 1;
  const int n_kv0 = q0_valid ? (p0s + last0) / 128 + 1 : 0;
  const int n_kv1 = q1_valid ? (p0s + min(Ls, q_row0 + qoff1 + 128) - 1) / 128 + 1 : 0;
  const int n_kv = max(n_kv0, n_kv1);

  const uint32_t bar0 = smem_u32(bars);
  const uint32_t q_full = bar0;
  auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + ATT_SLOTS + s); };
  auto s_full = [&](int t) { return bar0 + 8u * (1 + 2 * ATT_SLOTS + t); };
  auto s_free = [&](int t) { return bar0 + 8u * (3 + 2 * ATT_SLOTS + t); };
  auto p_full = [&](int t) { return bar0 + 8u * (5 + 2 * ATT_SLOTS + t); };
  auto pv_done = [&](int t) { return bar0 + 8u * (7 + 2 * ATT_SLOTS + t); };
  const uint32_t drain = bar0 + 8u * (9 + 2 * ATT_SLOTS);

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < ATT_SLOTS; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(s_free(t), 128);
      mbar_init(p_full(t), 128);
      mbar_init(pv_done(t), 1);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = tmem_base_sh;   // S_t at col 128 t, O_t at col 256 + 128 t
  WaitCtx wc{&abort_sh, p.status, p.limit_ns, 3};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last_fill[ATT_SLOTS];
      for (int s = 0; s < ATT_SLOTS; ++s) last_fill[s] = -1;
      const int nq = q1_valid ? 2 : (q0_valid ? 1 : 0);
      mbar_arrive_expect_tx(q_full, nq * nreg * ATT_REGION);
      for (int t = 0; t < nq; ++t)
        for (int r = 0; r < nreg; ++r) {
          const int col = (h0 + (hp ? t : 0)) * hd + r * 64, row = q_row0 + (t ? qoff1 : 0);
          if (p.tab != nullptr)
            tma_load_2d(smem_u32(sQ + t * ATT_TILE + r * ATT_REGION), &tmQ, q_full, col, row_base + row);
          else
            tma_load_3d(smem_u32(sQ + t * ATT_TILE + r * ATT_REGION), &tmQ, q_full, col, row, b);
        }
      const int zkv = b * p.nkv + g;
      for (int f = 0; f < 2 * n_kv; ++f) {   // fill f: K_{f/2} (f even) or V_{f/2} (f odd)
        const int s = f % ATT_SLOTS;
        if (!mbar_wait(kv_empty(s), ((f / ATT_SLOTS) & 1) ^ 1u, wc, 1)) break;
        const CUtensorMap* m = (f & 1) ? &tmV : &tmK;
        mbar_arrive_expect_tx(kv_full(s), nreg * ATT_REGION);
        for (int r = 0; r < nreg; ++r)
          tma_load_3d(smem_u32(sKV + s * ATT_TILE + r * ATT_REGION), m, kv_full(s), r * 64, (f >> 1) * 128, zkv);
        last_fill[s] = f;
      }
      // drain own copies before exit
      mbar_wait(q_full, 0, wc, 9, false);
      for (int s = 0; s < ATT_SLOTS; ++s)
        if (last_fill[s] >= 0) mbar_wait(kv_full(s), (last_fill[s] / ATT_SLOTS) & 1, wc, 9, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, hd_pad, 0, 1);   // V is MN-major
      const int ksteps = hd / 16;
      bool ok = mbar_wait(q_full, 0, wc, 2);
      bool issued = false;
      int s_count[2] = {0, 0};
      auto slot_ready = [&](int f) -> bool {   // wait for fill f of the ring
        return mbar_wait(kv_full(f % ATT_SLOTS), (f / ATT_SLOTS) & 1, wc, 3);
      };
      auto issue_s = [&](int t, int j) -> bool {
        if (!mbar_wait(s_free(t), (s_count[t] & 1) ^ 1u, wc, 4)) return false;
        tc_fence_after();
        const uint32_t aQ = smem_u32(sQ + t * ATT_TILE);
        const uint32_t aK = smem_u32(sKV + ((2 * j) % ATT_SLOTS) * ATT_TILE);
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t off = (ks >> 2) * ATT_REGION + (ks & 3) * 32;
          umma_bf16(tmem + t * 128, smem_desc_sw128(aQ + off, 16, 1024), smem_desc_sw128(aK + off, 16, 1024),
                    idesc_s, ks > 0 ? 1u : 0u);
        }
        umma_commit(s_full(t));
        ++s_count[t];
        issued = true;
        return true;
      };
      // O_t += P_t V_j with P_t the A operand in TMEM: bf16 pairs in the first 64
      // columns of S_t (written there by the softmax warps); issued before S_t's
      // next MMA, and tcgen05 MMAs run in order, so P is read before S is rewritten
      auto issue_pv = [&](int t, int j) -> bool {
        if (!mbar_wait(p_full(t), j & 1, wc, 5)) return false;
        tc_fence_after();
        const uint32_t aV = smem_u32(sKV + ((2 * j + 1) % ATT_SLOTS) * ATT_TILE);
        for (int ks = 0; ks < 8; ++ks) {   // 128 keys, 16 per MMA (8 TMEM columns of bf16 pairs)
          const uint32_t va = aV + ks * 16 * 128;
          umma_bf16_ts(tmem + 256 + t * 128, tmem + t * 128 + 8 * ks, smem_desc_sw128(va, ATT_REGION, 1024), idesc_o,
                       (j > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(pv_done(t));
        return true;
      };
      if (ok && n_kv0 > 0) ok = slot_ready(0) && issue_s(0, 0);
      for (int j = 0; ok && j < n_kv; ++j) {
        const bool a0 = j < n_kv0, a1 = j < n_kv1;
        if (a1) {
          if (!a0) ok = slot_ready(2 * j);   // K_j not waited for by tile 0
          if (ok) ok = issue_s(1, j);
        }
        if (!ok) break;
        umma_commit(kv_empty((2 * j) % ATT_SLOTS));          // K_j free once its S MMAs finish
        if (!slot_ready(2 * j + 1)) break;                  // V_j
        if (a0 && !issue_pv(0, j)) break;
        if (j + 1 < n_kv0 && !(slot_ready(2 * j + 2) && issue_s(0, j + 1))) break;
        if (a1 && !issue_pv(1, j)) break;
        umma_commit(kv_empty((2 * j + 1) % ATT_SLOTS));      // V_j free once its P·V MMAs finish
      }
      if (issued) {
        umma_commit(drain);
        mbar_wait(drain, 0, wc, 8, false);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / correction / epilogue
    const int t = (warp - 2) >> 2;             // query tile of this warpgroup
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int tok = q_row0 + (t ? qoff1 : 0) + row;   // token within the sequence
    const int pos = p0s + tok;
    const int pos_min = p0s + q_row0 + (t ? qoff1 : 0);
    const int h = h0 + (hp ? t : 0);                     // this tile's query head
    const int my_kv = t == 0 ? n_kv0 : n_kv1;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * 128;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < my_kv && ok; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(s_full(t), j & 1, wc, 10))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // all four 32-column loads in flight, one wait
      float sv[4][32];
      tmem_ld32(tS + 0, sv[0]);
      tmem_ld32(tS + 32, sv[1]);
      tmem_ld32(tS + 64, sv[2]);
      tmem_ld32(tS + 96, sv[3]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(s_free(t));
      // raw scores: the scale (> 0) is applied once to the maximum and folded
      // into the exponent below
      const bool need_mask = j * 128 + 127 > pos_min;
      if (need_mask) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (j * 128 + i > pos) sv[i >> 5][i & 31] = -INFINITY;
      }
      // four independent running maxima (exact in any order), then combined
      float mr[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) mr[k] = sv[0][k];
#pragma unroll
      for (int i = 4; i < 128; ++i) mr[i & 3] = fmaxf(mr[i & 3], sv[i >> 5][i & 31]);
      const float mraw = fmaxf(fmaxf(mr[0], mr[1]), fmaxf(mr[2], mr[3]));
      const float mx = mraw * p.scale_log2;
      // Move this row's reference maximum only when it grew by more than
      // 2^8; rows that keep theirs use alpha = 1.  The O rescale below is a
      // warp-collective TMEM read-modify-write, so the warp does it when any
      // of its rows needs it.
      float alpha = 1.f;
      const bool need = mx > m_used + 8.0f;
      if (need) {
        alpha = (m_used == -INFINITY) ? 0.f : ex2_approx(m_used - mx);
        m_used = mx;
      }
      const bool rescale = __any_sync(0xffffffffu, need && j > 0);
      // the previous P·V of this tile must be done (O stable, P buffer free)
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(pv_done(t), (j - 1) & 1, wc, 11))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // P = 2^(s - m_used) as bf16 pairs into this row's TMEM lane, over the
      // first 64 columns of S (already read into registers)
      const float mref = (m_used == -INFINITY) ? 0.f : m_used;
      const float sc = p.scale_log2;
      float ps[4] = {0.f, 0.f, 0.f, 0.f};   // four independent partial sums
#pragma unroll
      for (int g4 = 0; g4 < 4; ++g4) {   // keys 32 g4 .. 32 g4 + 31 -> columns 16 g4 .. 16 g4 + 15
        uint32_t pw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a = ex2_approx(fmaf(sv[g4][2 * e], sc, -mref));
          const float bb = ex2_approx(fmaf(sv[g4][2 * e + 1], sc, -mref));
          ps[e & 3] += a + bb;
          pw[e] = pack_bf16x2(a, bb);
        }
        tmem_st16u(tS + 16 * g4, pw);
      }
      // rescale O after P is written: the scores are dead by now, which keeps
      // the 128 loaded O columns from competing with them for registers
      if (rescale) {
        l *= alpha;
        if (hd_pad == 128) {
          float v0[32], v1[32], v2[32], v3[32];
          tmem_ld32(tO + 0, v0);
          tmem_ld32(tO + 32, v1);
          tmem_ld32(tO + 64, v2);
          tmem_ld32(tO + 96, v3);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            v0[i] *= alpha;
            v1[i] *= alpha;
            v2[i] *= alpha;
            v3[i] *= alpha;
          }
          tmem_st32(tO + 0, v0);
          tmem_st32(tO + 32, v1);
          tmem_st32(tO + 64, v2);
          tmem_st32(tO + 96, v3);
        } else {
          float v0[32], v1[32];
          tmem_ld32(tO + 0, v0);
          tmem_ld32(tO + 32, v1);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            v0[i] *= alpha;
            v1[i] *= alpha;
          }
          tmem_st32(tO + 0, v0);
          tmem_st32(tO + 32, v1);
        }
      }
      tmem_st_wait();   // P (and a rescaled O) in TMEM before the MMA warp is told
      l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      tc_fence_before();
      mbar_arrive(p_full(t));
    }
    if (ok && my_kv > 0 && __all_sync(0xffffffffu, mbar_wait(pv_done(t), (my_kv - 1) & 1, wc, 12))) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* orow = p.out + ((size_t)row_base + tok) * (size_t)(p.nh * hd) + (size_t)h * hd;
      for (int c = 0; c < hd_pad; c += 32) {
        float v[32];
        tmem_ld32(tO + c, v);
        tmem_ld_wait();
        if (tok < Ls) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (c + 8 * q < hd) {
              uint4 w;
              w.x = pack_bf16x2(v[8 * q + 0] * inv, v[8 * q + 1] * inv);
              w.y = pack_bf16x2(v[8 * q + 2] * inv, v[8 * q + 3] * inv);
              w.z = pack_bf16x2(v[8 * q + 4] * inv, v[8 * q + 5] * inv);
              w.w = pack_bf16x2(v[8 * q + 6] * inv, v[8 * q + 7] * inv);
              *reinterpret_cast<uint4*>(orow + c + 8 * q) = w;
            }
          }
        }
      }
    }
  }

  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// The same work split with the key axis advanced 64 keys per step.  Each query
// tile then has two S buffers of 64 TMEM columns (S_t at t * 128 + 64 (s & 1),
// O_t at 256 + 128 t, as before), so S_t(s + 1) is computed while the softmax
// works on S_t(s), and the softmax of one tile runs step after step instead of
// waiting for its own P·V and next S.  P_t(s) (bf16 pairs) goes over the first
// 32 columns of its S buffer.  The MMA warp issues, per step and tile, P·V of
// step s and then S of step s + 2 into the buffer P_t(s) came from: tcgen05
// MMAs of one thread run in order, so the P·V has read P before S overwrites
// it, and the softmax, having seen S_t(s) complete, knows that every P·V up
// to s - 2 has completed (a commit covers all earlier MMAs of its thread).
// The softmax waits for the previous P·V only to rescale O.  K / V arrive as
// 128-key tiles in the same 4-slot ring; step s reads rows 64 (s & 1) .. of
// tile s / 2.
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attn_prefill_k64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const AttnPrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                   // tile t at t * ATT_TILE
  uint8_t* sKV = sQ + 2 * ATT_TILE;                     // slot s at s * ATT_TILE
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + ATT_SLOTS * ATT_TILE);
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // heaviest query blocks first (grid.z), as in attn_prefill_kernel
  const int qb = p.n_qblocks - 1 - blockIdx.z;
  const int b = blockIdx.y;
  const bool hp = p.head_pair != 0;
  const int h0 = hp ? 2 * blockIdx.x : blockIdx.x;
  const int g = h0 / (p.nh / p.nkv);
  const int hd = p.hd;
  const int nreg = hd > 64 ? 2 : 1;
  const int hd_pad = nreg * 64;
  const int q_row0 = qb * (hp ? 128 : 256);
  const int qoff1 = hp ? 0 : 128;
  int Ls = p.L, p0s = p.p0, row_base = b * p.L;
  if (p.tab != nullptr) {
    pdl_wait();   // the table is written by an earlier kernel
    Ls = p.tab->len[b];
    p0s = p.tab->p0[b];
    row_base = p.tab->start[b];
  }
  const bool q0_valid = q_row0 < Ls;
  const bool q1_valid = q_row0 + qoff1 < Ls;
  // 64-key steps with any key visible to tile t (0 for an empty tile)
  const int n_st0 = q0_valid ? (p0s + min(Ls, q_row0 + 128) - 1) / 64 + 1 : 0;
  const int n_st1 = q1_valid ? (p0s + min(Ls, q_row0 + qoff1 + 128) - 1) / 64 + 1 : 0;
  const int n_st = max(n_st0, n_st1);
  const int n_kv = (n_st + 1) / 2;   // 128-key tiles to load

  const uint32_t bar0 = smem_u32(bars);
  const uint32_t q_full = bar0;
  auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + ATT_SLOTS + s); };
  // per tile t and S buffer u
  auto s_full = [&](int t, int u) { return bar0 + 8u * (1 + 2 * ATT_SLOTS + 2 * t + u); };
  auto p_full = [&](int t, int u) { return bar0 + 8u * (5 + 2 * ATT_SLOTS + 2 * t + u); };
  auto pv_done = [&](int t, int u) { return bar0 + 8u * (9 + 2 * ATT_SLOTS + 2 * t + u); };
  const uint32_t drain = bar0 + 8u * (13 + 2 * ATT_SLOTS);

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < ATT_SLOTS; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t)
      for (int u = 0; u < 2; ++u) {
        mbar_init(s_full(t, u), 1);
        mbar_init(p_full(t, u), 128);
        mbar_init(pv_done(t, u), 1);
      }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = tmem_base_sh;
  WaitCtx wc{&abort_sh, p.status, p.limit_ns, 3};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last_fill[ATT_SLOTS];
      for (int s = 0; s < ATT_SLOTS; ++s) last_fill[s] = -1;
      const int nq = q1_valid ? 2 : (q0_valid ? 1 : 0);
      mbar_arrive_expect_tx(q_full, nq * nreg * ATT_REGION);
      for (int t = 0; t < nq; ++t)
        for (int r = 0; r < nreg; ++r) {
          const int col = (h0 + (hp ? t : 0)) * hd + r * 64, row = q_row0 + (t ? qoff1 : 0);
          if (p.tab != nullptr)
            tma_load_2d(smem_u32(sQ + t * ATT_TILE + r * ATT_REGION), &tmQ, q_full, col, row_base + row);
          else
            tma_load_3d(smem_u32(sQ + t * ATT_TILE + r * ATT_REGION), &tmQ, q_full, col, row, b);
        }
      const int zkv = b * p.nkv + g;
      for (int f = 0; f < 2 * n_kv; ++f) {   // fill f: K_{f/2} (f even) or V_{f/2} (f odd)
        const int s = f % ATT_SLOTS;
        if (!mbar_wait(kv_empty(s), ((f / ATT_SLOTS) & 1) ^ 1u, wc, 1)) break;
        const CUtensorMap* m = (f & 1) ? &tmV : &tmK;
        mbar_arrive_expect_tx(kv_full(s), nreg * ATT_REGION);
        for (int r = 0; r < nreg; ++r)
          tma_load_3d(smem_u32(sKV + s * ATT_TILE + r * ATT_REGION), m, kv_full(s), r * 64, (f >> 1) * 128, zkv);
        last_fill[s] = f;
      }
      mbar_wait(q_full, 0, wc, 9, false);
      for (int s = 0; s < ATT_SLOTS; ++s)
        if (last_fill[s] >= 0) mbar_wait(kv_full(s), (last_fill[s] / ATT_SLOTS) & 1, wc, 9, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, hd_pad, 0, 1);   // V is MN-major
      const int ksteps = hd / 16;
      const int nst[2] = {n_st0, n_st1};
      bool ok = mbar_wait(q_full, 0, wc, 2);
      bool issued = false;
      auto fill_ready = [&](int f) -> bool {   // fill f of the ring has landed
        return mbar_wait(kv_full(f % ATT_SLOTS), (f / ATT_SLOTS) & 1, wc, 3);
      };
      // S_t(s) = Q_t K^T over keys 64 s .. 64 s + 63, into buffer s & 1
      auto issue_s = [&](int t, int s) -> bool {
        if (!fill_ready(2 * (s >> 1))) return false;
        tc_fence_after();
        const uint32_t aQ = smem_u32(sQ + t * ATT_TILE);
        const uint32_t aK = smem_u32(sKV + ((2 * (s >> 1)) % ATT_SLOTS) * ATT_TILE) + (uint32_t)((s & 1) * 64 * 128);
        const uint32_t d = tmem + (uint32_t)(t * 128 + (s & 1) * 64);
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t off = (ks >> 2) * ATT_REGION + (ks & 3) * 32;
          umma_bf16(d, smem_desc_sw128(aQ + off, 16, 1024), smem_desc_sw128(aK + off, 16, 1024), idesc_s,
                    ks > 0 ? 1u : 0u);
        }
        umma_commit(s_full(t, s & 1));
        issued = true;
        return true;
      };
      // O_t += P_t(s) V over the same 64 keys, P_t(s) the A operand in TMEM
      auto issue_pv = [&](int t, int s) -> bool {
        if (!mbar_wait(p_full(t, s & 1), (s >> 1) & 1, wc, 5)) return false;
        if (!fill_ready(2 * (s >> 1) + 1)) return false;
        tc_fence_after();
        const uint32_t aV =
            smem_u32(sKV + ((2 * (s >> 1) + 1) % ATT_SLOTS) * ATT_TILE) + (uint32_t)((s & 1) * 64 * 128);
        const uint32_t pa = tmem + (uint32_t)(t * 128 + (s & 1) * 64);
        for (int ks = 0; ks < 4; ++ks)   // 16 keys per MMA (8 TMEM columns of bf16 pairs)
          umma_bf16_ts(tmem + 256 + t * 128, pa + 8 * ks, smem_desc_sw128(aV + ks * 16 * 128, ATT_REGION, 1024),
                       idesc_o, (s > 0 || ks > 0) ? 1u : 0u);
        umma_commit(pv_done(t, s & 1));
        return true;
      };
      for (int s = 0; s < 2 && ok; ++s)
        for (int t = 0; t < 2 && ok; ++t)
          if (s < nst[t]) ok = issue_s(t, s);
      if (ok && n_st > 0) umma_commit(kv_empty(0));   // K_0: steps 0 and 1 issued
      for (int s = 0; ok && s < n_st; ++s) {
        for (int t = 0; t < 2 && ok; ++t) {
          if (s >= nst[t]) continue;
          ok = issue_pv(t, s);
          if (ok && s + 2 < nst[t]) ok = issue_s(t, s + 2);
        }
        if (!ok) break;
        if (s & 1) {
          // after step s (odd): V_{s/2} read by its last P·V, K_{(s+1)/2} by its last S
          umma_commit(kv_empty((2 * (s >> 1) + 1) % ATT_SLOTS));
          const int jk = (s + 1) >> 1;
          if (jk < n_kv) umma_commit(kv_empty((2 * jk) % ATT_SLOTS));
        }
      }
      if (issued) {
        umma_commit(drain);
        mbar_wait(drain, 0, wc, 8, false);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / correction / epilogue
    const int t = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int tok = q_row0 + (t ? qoff1 : 0) + row;
    const int pos = p0s + tok;
    const int pos_min = p0s + q_row0 + (t ? qoff1 : 0);
    const int h = h0 + (hp ? t : 0);
    const int my_st = t == 0 ? n_st0 : n_st1;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * 128;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int s = 0; s < my_st && ok; ++s) {
      const int u = s & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full(t, u), (s >> 1) & 1, wc, 10))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[2][32];
      tmem_ld32(tS + u * 64, sv[0]);
      tmem_ld32(tS + u * 64 + 32, sv[1]);
      tmem_ld_wait();
      if (s * 64 + 63 > pos_min) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (s * 64 + i > pos) sv[i >> 5][i & 31] = -INFINITY;
      }
      float mr[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) mr[k] = sv[0][k];
#pragma unroll
      for (int i = 4; i < 64; ++i) mr[i & 3] = fmaxf(mr[i & 3], sv[i >> 5][i & 31]);
      const float mx = fmaxf(fmaxf(mr[0], mr[1]), fmaxf(mr[2], mr[3])) * p.scale_log2;
      // the reference maximum moves only when it grew by more than 2^8
      float alpha = 1.f;
      const bool need = mx > m_used + 8.0f;
      if (need) {
        alpha = (m_used == -INFINITY) ? 0.f : ex2_approx(m_used - mx);
        m_used = mx;
      }
      const bool rescale = __any_sync(0xffffffffu, need && s > 0);
      const float mref = (m_used == -INFINITY) ? 0.f : m_used;
      const float sc = p.scale_log2;
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pw[2][16];
#pragma unroll
      for (int g2 = 0; g2 < 2; ++g2)
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a = ex2_approx(fmaf(sv[g2][2 * e], sc, -mref));
          const float bb = ex2_approx(fmaf(sv[g2][2 * e + 1], sc, -mref));
          ps[e & 3] += a + bb;
          pw[g2][e] = pack_bf16x2(a, bb);
        }
      tmem_st16u(tS + u * 64, pw[0]);
      tmem_st16u(tS + u * 64 + 16, pw[1]);
      if (rescale) {
        // O must hold every earlier step: wait for P·V of step s - 1 (those up
        // to s - 2 completed before S_t(s), which the wait above saw)
        if (!__all_sync(0xffffffffu, mbar_wait(pv_done(t, u ^ 1), ((s - 1) >> 1) & 1, wc, 11))) {
          ok = false;
          break;
        }
        tc_fence_after();
        l *= alpha;
        if (hd_pad == 128) {
          float v0[32], v1[32], v2[32], v3[32];
          tmem_ld32(tO + 0, v0);
          tmem_ld32(tO + 32, v1);
          tmem_ld32(tO + 64, v2);
          tmem_ld32(tO + 96, v3);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            v0[i] *= alpha;
            v1[i] *= alpha;
            v2[i] *= alpha;
            v3[i] *= alpha;
          }
          tmem_st32(tO + 0, v0);
          tmem_st32(tO + 32, v1);
          tmem_st32(tO + 64, v2);
          tmem_st32(tO + 96, v3);
        } else {
          float v0[32], v1[32];
          tmem_ld32(tO + 0, v0);
          tmem_ld32(tO + 32, v1);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            v0[i] *= alpha;
            v1[i] *= alpha;
          }
          tmem_st32(tO + 0, v0);
          tmem_st32(tO + 32, v1);
        }
      }
      tmem_st_wait();   // P (and a rescaled O) in TMEM before the MMA warp is told
      l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      tc_fence_before();
      mbar_arrive(p_full(t, u));
    }
    // the last P·V (those before it completed before the last S)
    const int sl = my_st - 1;
    if (ok && my_st > 0 && __all_sync(0xffffffffu, mbar_wait(pv_done(t, sl & 1), (sl >> 1) & 1, wc, 12))) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* orow = p.out + ((size_t)row_base + tok) * (size_t)(p.nh * hd) + (size_t)h * hd;
      for (int c = 0; c < hd_pad; c += 32) {
        float v[32];
        tmem_ld32(tO + c, v);
        tmem_ld_wait();
        if (tok < Ls) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (c + 8 * q < hd) {
              uint4 w;
              w.x = pack_bf16x2(v[8 * q + 0] * inv, v[8 * q + 1] * inv);
              w.y = pack_bf16x2(v[8 * q + 2] * inv, v[8 * q + 3] * inv);
              w.z = pack_bf16x2(v[8 * q + 4] * inv, v[8 * q + 5] * inv);
              w.w = pack_bf16x2(v[8 * q + 6] * inv, v[8 * q + 7] * inv);
              *reinterpret_cast<uint4*>(orow + c + 8 * q) = w;
            }
          }
        }
      }
    }
  }

  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ====================================================================== decode

struct AttnDecodeParams {
  const __nv_bfloat16* qkv;   // [B, ld_qkv], q heads at columns h*hd (already rotated)
  int ld_qkv;
  const __nv_bfloat16* kc;    // [B][nkv][cap][hd]
  const __nv_bfloat16* vc;
  int cap, T;                 // capacity, visible keys (cache length after the append)
  int nh, nkv;
  int splits, keys_per_split;
  float scale_log2;
  float* part_ml;             // [B*nh][splits][2]   (splits > 1)
  float* part_o;              // [B*nh][splits][hd]
  __nv_bfloat16* out;         // [B, nh*hd]
  const SeqTab* tab;          // ragged: sequence b sees tab->p0[b] + 1 keys; nullptr: all see T
  // RoPE + KV append fused in (one key split): qkv holds the raw projections;
  // the kernel rotates q and the new k at position T - 1, appends k and v to the
  // cache there and writes the rotated q back into qkv
  float theta;
  int rope_style;
};

// Log-sum-exp merge of the `splits` partial results of query head hq of
// sequence b (base-2 maxima): out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
// Partials are read through L2: other CTAs of the same launch may have written them.
__device__ __forceinline__ void combine_head(const float* part_ml, const float* part_o, __nv_bfloat16* out, int nh,
                                             int hd, int splits, int b, int hq) {
  const size_t r0 = ((size_t)b * nh + hq) * splits;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, __ldcg(part_ml + 2 * (r0 + s)));
  for (int d = threadIdx.x; d < hd; d += blockDim.x) {
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
      for (int s = 0; s < splits; ++s) {
        const float c = exp2f(__ldcg(part_ml + 2 * (r0 + s)) - M);
        Lsum += __ldcg(part_ml + 2 * (r0 + s) + 1) * c;
        O += __ldcg(part_o + (r0 + s) * hd + d) * c;
      }
    }
    out[(size_t)b * nh * hd + (size_t)hq * hd + d] = __float2bfloat16_rn(Lsum > 0.f ? O / Lsum : 0.f);
  }
}


// Lane slice [sub * VEC, sub * VEC + VEC) of one head row (bf16) -> fp32,
// read through L2 (the row may have been written by another CTA of the same
// kernel).
template <int VEC>
__device__ __forceinline__ void load_slice(const __nv_bfloat16* src, float (&x)[VEC]) {
#pragma unroll
  for (int v = 0; v < VEC / 8; ++v) {
    uint4 u = __ldcg(reinterpret_cast<const uint4*>(src + 8 * v));
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      x[8 * v + 2 * e] = f.x;
      x[8 * v + 2 * e + 1] = f.y;
    }
  }
}

// RoPE of one lane's slice (dims sub*VEC ...) of a head row, rounded to bf16
// as the stand-alone RoPE kernel stores it: rotate-half pairs d with d + HD/2
// (held by lane sub ^ LPK/2 of the same key group), interleaved pairs (2i, 2i+1)
// within the slice; cs/sn: the position's cos/sin per pair index.
template <int HD, int LPK, int VEC>
__device__ __forceinline__ void rope_slice(float (&x)[VEC], int sub, int style, const float* cs, const float* sn) {
  if (style == 0) {
    const bool lower = sub < LPK / 2;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, x[e], LPK / 2);
      const int d = sub * VEC + e, i = lower ? d : d - HD / 2;
      const float c = cs[i], s = sn[i];
      x[e] = lower ? rope_lo(x[e], other, c, s) : rope_hi(other, x[e], c, s);
    }
  } else {
#pragma unroll
    for (int e = 0; e < VEC; e += 2) {
      const int i = (sub * VEC + e) >> 1;
      const float c = cs[i], s = sn[i], x0 = x[e], x1 = x[e + 1];
      x[e] = rope_lo(x0, x1, c, s);
      x[e + 1] = rope_hi(x0, x1, c, s);
    }
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) x[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
}

template <int VEC>
__device__ __forceinline__ void store_slice(__nv_bfloat16* dst, const float (&x)[VEC]) {
#pragma unroll
  for (int v = 0; v < VEC / 8; ++v) {
    uint4 w;
    w.x = pack_bf16x2(x[8 * v + 0], x[8 * v + 1]);
    w.y = pack_bf16x2(x[8 * v + 2], x[8 * v + 3]);
    w.z = pack_bf16x2(x[8 * v + 4], x[8 * v + 5]);
    w.w = pack_bf16x2(x[8 * v + 6], x[8 * v + 7]);
    *reinterpret_cast<uint4*>(dst + 8 * v) = w;
  }
}

// Shared memory of one 128-thread decode-attention group.
template <int HD, int G>
struct DecAttnSmem {
  float rcs[HD / 2], rsn[HD / 2];   // RoPE: cos / sin of the new token's angles
  float m[4][G], l[4][G];           // per-warp softmax state
  float o[4][G][HD];
};

// The new token's RoPE angles (position: the cache length before this step).
template <int HD, int G>
__device__ __forceinline__ void dec_attn_angles(const AttnDecodeParams& p, int b, int tid, DecAttnSmem<HD, G>& sh) {
  const int pos = p.tab != nullptr ? p.tab->p0[b] : p.T - 1;
  for (int i = tid; i < HD / 2; i += 128) rope_cos_sin(pos, i, HD, p.theta, sh.rcs[i], sh.rsn[i]);
}

// Decode attention of (key split `split`, KV head g, sequence b), run by 128
// threads (tid 0..127, four whole warps) that meet at `sync`.  ROPE: the
// angles must be in sh.rcs / sh.rsn before the call (dec_attn_angles).
template <int HD, int G, bool ROPE, typename Sync>
__device__ __forceinline__ void attn_decode_body(const AttnDecodeParams& p, int split, int g, int b, int tid,
                                                 DecAttnSmem<HD, G>& sh, Sync&& sync) {
  constexpr int LPK = HD == 96 ? 4 : HD / 8;    // lanes per key (power of two)
  constexpr int VEC = HD / LPK;                 // elements per lane
  constexpr int NV = VEC / 8;                   // 16-byte loads per lane per row
  constexpr int KPW = 32 / LPK;                 // keys per warp step
  constexpr int NK = 4;                         // keys per lane group per step
  constexpr int NW = 4;
  const float* rcs = sh.rcs;
  const float* rsn = sh.rsn;
  const int warp = tid >> 5, lane = tid & 31;
  const int grp = lane / LPK, sub = lane % LPK;
  const int T = p.tab != nullptr ? p.tab->p0[b] + 1 : p.T;
  const int j0 = split * p.keys_per_split;
  const int j1 = min(T, j0 + p.keys_per_split);
  const int j1c = ROPE ? min(j1, T - 1) : j1;   // keys read from the cache

  float q[G][VEC];
  const __nv_bfloat16* row = p.qkv + (size_t)b * p.ld_qkv;
#pragma unroll
  for (int gi = 0; gi < G; ++gi) {
    load_slice<VEC>(row + (size_t)(g * G + gi) * HD + sub * VEC, q[gi]);
    if (ROPE) rope_slice<HD, LPK, VEC>(q[gi], sub, p.rope_style, rcs, rsn);
  }
  float kn[VEC], vn[VEC];   // the new token's rotated key and value (ROPE)
  if (ROPE) {
    load_slice<VEC>(row + (size_t)(p.nh + g) * HD + sub * VEC, kn);
    load_slice<VEC>(row + (size_t)(p.nh + p.nkv + g) * HD + sub * VEC, vn);
    rope_slice<HD, LPK, VEC>(kn, sub, p.rope_style, rcs, rsn);
    sync();   // every thread has read the raw q before it is overwritten
    if (warp == 0 && grp == 0) {
      const int pos = T - 1;
      const size_t c = (((size_t)b * p.nkv + g) * p.cap + pos) * HD + sub * VEC;
      store_slice<VEC>(const_cast<__nv_bfloat16*>(p.kc) + c, kn);
      store_slice<VEC>(const_cast<__nv_bfloat16*>(p.vc) + c, vn);
#pragma unroll
      for (int gi = 0; gi < G; ++gi)
        store_slice<VEC>(const_cast<__nv_bfloat16*>(row) + (size_t)(g * G + gi) * HD + sub * VEC, q[gi]);
    }
  }
#pragma unroll
  for (int gi = 0; gi < G; ++gi)
#pragma unroll
    for (int e = 0; e < VEC; ++e) q[gi][e] *= p.scale_log2;
  float m[G], l[G], o[G][VEC];
#pragma unroll
  for (int gi = 0; gi < G; ++gi) {
    m[gi] = -INFINITY;
    l[gi] = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) o[gi][e] = 0.f;
  }
  const size_t head_off = ((size_t)b * p.nkv + g) * (size_t)p.cap * HD + sub * VEC;
  const __nv_bfloat16* K = p.kc + head_off;
  const __nv_bfloat16* V = p.vc + head_off;
  constexpr int STEP = NW * KPW * NK;
  for (int wb = j0 + warp * KPW * NK; wb < j1c; wb += STEP) {
    uint4 kr[NK][NV], vr[NK][NV];
#pragma unroll
    for (int kk = 0; kk < NK; ++kk) {
      const int j = wb + grp * NK + kk;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        if (j < j1c) {
          kr[kk][v] = __ldg(reinterpret_cast<const uint4*>(K + (size_t)j * HD) + v);
          vr[kk][v] = __ldg(reinterpret_cast<const uint4*>(V + (size_t)j * HD) + v);
        } else {
          kr[kk][v] = make_uint4(0, 0, 0, 0);
          vr[kk][v] = make_uint4(0, 0, 0, 0);
        }
      }
    }
    float s[NK][G];
#pragma unroll
    for (int kk = 0; kk < NK; ++kk) {
      float kf[VEC];
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&kr[kk][v]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          kf[8 * v + 2 * e] = f.x;
          kf[8 * v + 2 * e + 1] = f.y;
        }
      }
#pragma unroll
      for (int gi = 0; gi < G; ++gi) {
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) d = fmaf(q[gi][e], kf[e], d);
#pragma unroll
        for (int off = LPK / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        s[kk][gi] = (wb + grp * NK + kk < j1c) ? d : -INFINITY;
      }
    }
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      float mx = s[0][gi];
#pragma unroll
      for (int kk = 1; kk < NK; ++kk) mx = fmaxf(mx, s[kk][gi]);
      const float mn = fmaxf(m[gi], mx);
      if (mn == -INFINITY) continue;
      const float alpha = exp2f(m[gi] - mn);
      m[gi] = mn;
      l[gi] *= alpha;
#pragma unroll
      for (int e = 0; e < VEC; ++e) o[gi][e] *= alpha;
#pragma unroll
      for (int kk = 0; kk < NK; ++kk) {
        const float pk = exp2f(s[kk][gi] - mn);
        l[gi] += pk;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&vr[kk][v]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            o[gi][8 * v + 2 * e] = fmaf(pk, f.x, o[gi][8 * v + 2 * e]);
            o[gi][8 * v + 2 * e + 1] = fmaf(pk, f.y, o[gi][8 * v + 2 * e + 1]);
          }
        }
      }
    }
  }
  if (ROPE && j1 == T && warp == 0) {
    // the new key (position T - 1) from registers, in lane group 0 of warp 0
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) d = fmaf(q[gi][e], kn[e], d);
#pragma unroll
      for (int off = LPK / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
      if (grp == 0) {
        const float mn = fmaxf(m[gi], d);
        const float alpha = exp2f(m[gi] - mn), pk = exp2f(d - mn);
        m[gi] = mn;
        l[gi] = l[gi] * alpha + pk;
#pragma unroll
        for (int e = 0; e < VEC; ++e) o[gi][e] = fmaf(pk, vn[e], o[gi][e] * alpha);
      }
    }
  }
  // merge the lane groups of the warp (same `sub`, different keys)
#pragma unroll
  for (int off = LPK; off < 32; off <<= 1) {
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[gi], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l[gi], off);
      const float mn = fmaxf(m[gi], mo);
      const float a = mn == -INFINITY ? 0.f : exp2f(m[gi] - mn);
      const float c = mn == -INFINITY ? 0.f : exp2f(mo - mn);
      l[gi] = l[gi] * a + lo * c;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float oo = __shfl_xor_sync(0xffffffffu, o[gi][e], off);
        o[gi][e] = o[gi][e] * a + oo * c;
      }
      m[gi] = mn;
    }
  }
  // merge the warps through shared memory
  float (*sm_m)[G] = sh.m;
  float (*sm_l)[G] = sh.l;
  float (*sm_o)[G][HD] = sh.o;
  if (grp == 0) {
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      if (sub == 0) {
        sm_m[warp][gi] = m[gi];
        sm_l[warp][gi] = l[gi];
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) sm_o[warp][gi][sub * VEC + e] = o[gi][e];
    }
  }
  sync();
  for (int idx = tid; idx < G * HD; idx += 128) {
    const int gi = idx / HD, d = idx % HD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sm_m[w][gi]);
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float c = exp2f(sm_m[w][gi] - M);
        Lsum += sm_l[w][gi] * c;
        O += sm_o[w][gi][d] * c;
      }
    }
    const int hq = g * G + gi;
    if (p.splits == 1) {
      p.out[(size_t)b * p.nh * HD + (size_t)hq * HD + d] = __float2bfloat16_rn(Lsum > 0.f ? O / Lsum : 0.f);
    } else {
      const size_t r = ((size_t)b * p.nh + hq) * p.splits + split;
      p.part_o[r * HD + d] = O;
      if (d == 0) {
        p.part_ml[2 * r] = M;
        p.part_ml[2 * r + 1] = Lsum;
      }
    }
  }
}

template <int HD, int G, bool ROPE>
__global__ void __launch_bounds__(128) attn_decode_kernel(const AttnDecodeParams p) {
  __shared__ DecAttnSmem<HD, G> sh;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  // a ragged table is written by an earlier kernel, so its angles wait for it
  if (ROPE && p.tab == nullptr) dec_attn_angles<HD, G>(p, b, threadIdx.x, sh);
  pdl_wait();
  if (ROPE && p.tab != nullptr) dec_attn_angles<HD, G>(p, b, threadIdx.x, sh);
  if (ROPE) __syncthreads();
  attn_decode_body<HD, G, ROPE>(p, split, g, b, threadIdx.x, sh, [] { __syncthreads(); });
}

// ---------------------------------------------------------------------- decode, GQA groups >= 4
// The G query heads of a KV head are the rows of a 16-row MMA tile (rows
// G..15 are zero), so S = Q K^T and O += P V run on the tensor cores
// (mma.sync m16n8k16, bf16 -> fp32) and the kernel stays bound by the K/V
// stream.  One producer warp stages 64-key chunks of K and V by TMA (128-byte
// swizzle, 3-D maps over [head_dim, length, batch*n_kv]); one consumer warp
// per stage takes the chunks of its stage, each with its own online-softmax
// state; the warps' states are merged through shared memory at the end.

constexpr int DEC_CHUNK = 64;                          // keys per chunk
constexpr int DEC_REGION = DEC_CHUNK * 128;            // [64 keys x 64 dims] bf16 = 8 KB

// HD: head dimension as laid out in shared memory (64 or 128); a head_dim of 96
// runs as 128 with dims 96..127 zero-filled by the TMA bounds (no HBM bytes).
// STAGES: K/V chunks in flight (3 at HD 128 keeps two CTAs on an SM).
template <int HD, int STAGES_ = 4>
struct DecMmaCfg {
  static constexpr int STAGES = STAGES_;
  static constexpr int NREG = HD / 64;                 // 64-dim regions per key row
  static constexpr int STAGE = 2 * NREG * DEC_REGION;  // K then V
  static constexpr int SMEM = 1024 + STAGES * STAGE + 256;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of (key, 16-byte chunk) inside a swizzled [64 keys x 128 B] region
__device__ __forceinline__ uint32_t sw128(int key, int chunk) {
  return (uint32_t)(key * 128 + ((chunk ^ (key & 7)) << 4));
}

struct AttnDecodeMmaParams {
  const __nv_bfloat16* qkv;
  int ld_qkv;
  int hd;                     // head_dim in memory (<= the kernel's HD; 96 runs as 128)
  int T;
  int nh, nkv;
  int splits, keys_per_split;
  float scale_log2;
  float* part_ml;
  float* part_o;
  __nv_bfloat16* out;
  DevStatus* status;
  unsigned long long limit_ns;
  const SeqTab* tab;          // ragged: sequence b sees tab->p0[b] + 1 keys; nullptr: all see T
  // RoPE + KV append fused in (one key split; see AttnDecodeParams)
  __nv_bfloat16* kc;          // the caches, for the append of the new token's row
  __nv_bfloat16* vc;
  int cap;
  float theta;
  int rope_style;
};

// RoPE of the new token (position pos) for KV head g of sequence b, by one
// warp: the G query heads are rotated in place in qkv, the rotated key and the
// value go to cache row pos.  Rounds like the stand-alone RoPE kernel.
// cs / sn: the position's angles (dec_rope_angles_warp, then __syncwarp).
__device__ __forceinline__ void dec_rope_angles_warp(const AttnDecodeMmaParams& p, int pos, float* cs, float* sn) {
  for (int i = (int)(threadIdx.x & 31); i < (p.hd >> 1); i += 32) rope_cos_sin(pos, i, p.hd, p.theta, cs[i], sn[i]);
}

template <int G>
__device__ __forceinline__ void dec_rope_append_warp(const AttnDecodeMmaParams& p, int b, int g, int pos,
                                                     const float* cs, const float* sn) {
  const int lane = threadIdx.x & 31, hd = p.hd, half = hd >> 1;
  __nv_bfloat16* row = const_cast<__nv_bfloat16*>(p.qkv) + (size_t)b * p.ld_qkv;
  const size_t crow = (((size_t)b * p.nkv + g) * p.cap + pos) * hd;
  for (int h = 0; h <= G; ++h) {   // the G query heads, then the key head
    __nv_bfloat16* src = row + (size_t)(h < G ? g * G + h : p.nh + g) * hd;
    __nv_bfloat16* dst = h < G ? src : p.kc + crow;
    for (int i = lane; i < half; i += 32) {
      // rotate-half pairs (i, i + hd/2), interleaved pairs (2i, 2i + 1)
      const int i0 = p.rope_style == 0 ? i : 2 * i, i1 = p.rope_style == 0 ? i + half : 2 * i + 1, pi = i;
      // each pair is read and written by one lane, so q can rotate in place
      const float x0 = __bfloat162float(src[i0]), x1 = __bfloat162float(src[i1]);
      const float c = cs[pi], s = sn[pi];
      dst[i0] = __float2bfloat16_rn(rope_lo(x0, x1, c, s));
      dst[i1] = __float2bfloat16_rn(rope_hi(x0, x1, c, s));
    }
  }
  const __nv_bfloat16* v = row + (size_t)(p.nh + p.nkv + g) * hd;
  for (int i = lane; i < hd; i += 32) p.vc[crow + i] = v[i];
  __syncwarp();
}

// ST stages and ST consumer warps: warp w takes chunks w, w + ST, ... so each
// stage has one consumer, and its full / empty phases alternate in chunk order.
// ROPE (one key split): qkv holds the raw projections.  The producer warp
// computes the angles before the PDL wait, puts the chunks that do not hold
// the new token's row in flight, rotates q and the new key and appends the new
// k / v row, and only then loads the last chunk (which holds that row).
template <int HD, int G, int ST, bool ROPE>
__global__ void __launch_bounds__(32 * (ST + 1), 1)
    attn_decode_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const AttnDecodeMmaParams p) {
  using C = DecMmaCfg<HD, ST>;
  constexpr int DEC_STAGES = C::STAGES;
  constexpr int NW = ST;               // consumer warps, one per stage
  constexpr int KS = HD / 16;          // k-steps of S = Q K^T
  constexpr int NT_O = HD / 8;         // 8-dim output tiles
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DEC_STAGES * C::STAGE);
  __shared__ int abort_sh;
  __shared__ float sm_m[NW][16], sm_l[NW][16];
  __shared__ float sm_o[NW][G][HD];

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float rcs[ROPE ? HD / 2 : 1], rsn[ROPE ? HD / 2 : 1];
  // the new token's angles overlap the previous kernel (position known up front)
  if (ROPE && p.tab == nullptr && warp == 0) dec_rope_angles_warp(p, p.T - 1, rcs, rsn);
  if (p.tab != nullptr) pdl_wait();   // the ragged table is written by an earlier kernel
  const int T = p.tab != nullptr ? p.tab->p0[b] + 1 : p.T;
  if (ROPE && p.tab != nullptr && warp == 0) dec_rope_angles_warp(p, T - 1, rcs, rsn);
  const int j0 = split * p.keys_per_split;
  const int j1 = min(T, j0 + p.keys_per_split);
  const int n_chunks = j1 > j0 ? (j1 - j0 + DEC_CHUNK - 1) / DEC_CHUNK : 0;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (DEC_STAGES + s); };
  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < DEC_STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();
  WaitCtx wc{&abort_sh, p.status, p.limit_ns, 4};
  const int zkv = b * p.nkv + g;
  int last_fill[DEC_STAGES];
  for (int s = 0; s < DEC_STAGES; ++s) last_fill[s] = -1;
  int c_next = 0;   // producer: the next chunk to fill
  auto fill = [&](int c) -> bool {
    const int s = c % DEC_STAGES;
    if (!mbar_wait(empty_bar(s), ((c / DEC_STAGES) & 1) ^ 1u, wc, 1)) return false;
    uint8_t* st = smem + s * C::STAGE;
    mbar_arrive_expect_tx(full_bar(s), C::STAGE);
    const int key0 = j0 + c * DEC_CHUNK;
    for (int r = 0; r < C::NREG; ++r) {
      tma_load_3d(smem_u32(st + r * DEC_REGION), &tmK, full_bar(s), r * 64, key0, zkv);
      tma_load_3d(smem_u32(st + (C::NREG + r) * DEC_REGION), &tmV, full_bar(s), r * 64, key0, zkv);
    }
    last_fill[s] = c;
    return true;
  };
  if (ROPE) {
    if (warp == 0) {
      if (lane == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        // the chunks before the one holding row T - 1 do not depend on this step
        while (c_next < min(DEC_STAGES, n_chunks - 1) && fill(c_next)) ++c_next;
      }
      __syncwarp();
      dec_rope_append_warp<G>(p, b, g, T - 1, rcs, rsn);
    }
    __syncthreads();   // the consumers read the rotated q; the new row is written
  }

  if (warp == 0) {
    if (lane == 0) {
      if (ROPE) {
        // the new row was written by the warp's lanes through the generic proxy
        // (ordered before this thread by the barrier); the fills read it by TMA
        asm volatile("fence.proxy.async.global;" ::: "memory");
      } else {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      while (c_next < n_chunks && fill(c_next)) ++c_next;
      for (int s = 0; s < DEC_STAGES; ++s)
        if (last_fill[s] >= 0) mbar_wait(full_bar(s), (last_fill[s] / DEC_STAGES) & 1, wc, 9, false);
    }
  } else {
    const int cw = warp - 1;
    const int r0 = lane >> 2, qd = lane & 3;   // fragment row (and row + 8), quad position
    // Q as A fragments: rows = query heads of the group (rows >= G are zero)
    uint32_t qa[KS][4];
    {
      const int hdm = p.hd;
      const __nv_bfloat16* qrow0 = p.qkv + (size_t)b * p.ld_qkv + (size_t)(g * G) * hdm;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int k0 = ks * 16 + qd * 2;
        uint32_t lo = 0, hi = 0, lo8 = 0, hi8 = 0;
        // dims past head_dim stay zero (head_dim is a multiple of 16 here)
        // through L2: with ROPE the row was just rewritten by this CTA's producer warp
        if (r0 < G && k0 < hdm) {
          lo = __ldcg(reinterpret_cast<const unsigned int*>(qrow0 + (size_t)r0 * hdm + k0));
          lo8 = __ldcg(reinterpret_cast<const unsigned int*>(qrow0 + (size_t)r0 * hdm + k0 + 8));
        }
        if (r0 + 8 < G && k0 < hdm) {
          hi = __ldcg(reinterpret_cast<const unsigned int*>(qrow0 + (size_t)(r0 + 8) * hdm + k0));
          hi8 = __ldcg(reinterpret_cast<const unsigned int*>(qrow0 + (size_t)(r0 + 8) * hdm + k0 + 8));
        }
        qa[ks][0] = lo;
        qa[ks][1] = hi;
        qa[ks][2] = lo8;
        qa[ks][3] = hi8;
      }
    }
    float o[NT_O][4];
#pragma unroll
    for (int i = 0; i < NT_O; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;   // rows r0, r0 + 8
    bool ok = true;
    for (int c = cw; c < n_chunks && ok; c += NW) {
      const int s = c % DEC_STAGES;
      if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), (c / DEC_STAGES) & 1, wc, 2))) {
        ok = false;
        break;
      }
      const uint32_t sK = smem_u32(smem + s * C::STAGE);
      const uint32_t sV = sK + C::NREG * DEC_REGION;
      // S = Q K^T for 64 keys: 8 n-tiles of 8 keys
      float sc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        const int key = nt * 8 + (lane & 7);
#pragma unroll
        for (int kp = 0; kp < KS; kp += 2) {   // two k-steps (32 dims) per ldmatrix.x4
          const int chunk = kp * 2 + (lane >> 3);          // 16-byte chunk within the 256-byte row
          const uint32_t addr = sK + (chunk >> 3) * DEC_REGION + sw128(key, chunk & 7);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(addr, b0, b1, b2, b3);
          mma_bf16_16816(sc[nt], qa[kp], b0, b1);
          mma_bf16_16816(sc[nt], qa[kp + 1], b2, b3);
        }
      }
      // online softmax (log2 domain); keys outside [j0, j1) are masked
      const int kbase = j0 + c * DEC_CHUNK;
      float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool valid = kbase + nt * 8 + qd * 2 + e < j1;
          sc[nt][e] = valid ? sc[nt][e] * p.scale_log2 : -INFINITY;
          sc[nt][2 + e] = valid ? sc[nt][2 + e] * p.scale_log2 : -INFINITY;
          mx_a = fmaxf(mx_a, sc[nt][e]);
          mx_b = fmaxf(mx_b, sc[nt][2 + e]);
        }
      }
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
      const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
      const float al_a = mn_a == -INFINITY ? 1.f : ex2_approx(m_a - mn_a);
      const float al_b = mn_b == -INFINITY ? 1.f : ex2_approx(m_b - mn_b);
      m_a = mn_a;
      m_b = mn_b;
      const float ref_a = mn_a == -INFINITY ? 0.f : mn_a, ref_b = mn_b == -INFINITY ? 0.f : mn_b;
      l_a *= al_a;
      l_b *= al_b;
#pragma unroll
      for (int i = 0; i < NT_O; ++i) {
        o[i][0] *= al_a;
        o[i][1] *= al_a;
        o[i][2] *= al_b;
        o[i][3] *= al_b;
      }
      uint32_t pa[4][4];   // P as A fragments: 4 k-steps of 16 keys
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = ex2_approx(sc[nt][0] - ref_a), p1 = ex2_approx(sc[nt][1] - ref_a);
        const float p2 = ex2_approx(sc[nt][2] - ref_b), p3 = ex2_approx(sc[nt][3] - ref_b);
        l_a += p0 + p1;
        l_b += p2 + p3;
        pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(p0, p1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(p2, p3);
      }
      // O += P V: V rows are keys; ldmatrix.trans gives the k-major B fragments
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int key = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
        for (int dt = 0; dt < NT_O; dt += 2) {
          const int chunk = dt + (lane >> 4);              // 8-dim chunk index within the row
          const uint32_t addr = sV + (chunk >> 3) * DEC_REGION + sw128(key, chunk & 7);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(addr, b0, b1, b2, b3);
          mma_bf16_16816(o[dt], pa[kk], b0, b1);
          mma_bf16_16816(o[dt + 1], pa[kk], b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));
    }
    // quad-reduce the sums, then publish this warp's state
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    if (qd == 0) {
      sm_m[cw][r0] = m_a;
      sm_l[cw][r0] = l_a;
      sm_m[cw][r0 + 8] = m_b;
      sm_l[cw][r0 + 8] = l_b;
    }
#pragma unroll
    for (int dt = 0; dt < NT_O; ++dt) {
      const int col = dt * 8 + qd * 2;
      if (r0 < G) {
        sm_o[cw][r0][col] = o[dt][0];
        sm_o[cw][r0][col + 1] = o[dt][1];
      }
      if (r0 + 8 < G) {
        sm_o[cw][r0 + 8][col] = o[dt][2];
        sm_o[cw][r0 + 8][col + 1] = o[dt][3];
      }
    }
  }
  __syncthreads();
  pdl_trigger();
  const int hdm = p.hd;
  for (int idx = threadIdx.x; idx < G * hdm; idx += blockDim.x) {
    const int gi = idx / hdm, d = idx % hdm;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sm_m[w][gi]);
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float cf = exp2f(sm_m[w][gi] - M);
        Lsum += sm_l[w][gi] * cf;
        O += sm_o[w][gi][d] * cf;
      }
    }
    const int hq = g * G + gi;
    if (p.splits == 1) {
      p.out[(size_t)b * p.nh * hdm + (size_t)hq * hdm + d] = __float2bfloat16_rn(Lsum > 0.f ? O / Lsum : 0.f);
    } else {
      const size_t r = ((size_t)b * p.nh + hq) * p.splits + split;
      p.part_o[r * hdm + d] = O;
      if (d == 0) {
        p.part_ml[2 * r] = M;
        p.part_ml[2 * r + 1] = Lsum;
      }
    }
  }
}

// out[b, h*hd + d] = sum_s 2^(m_s - M) o_s[d] / sum_s 2^(m_s - M) l_s
__global__ void attn_decode_combine_kernel(const float* __restrict__ part_ml, const float* __restrict__ part_o,
                                           __nv_bfloat16* __restrict__ out, int nh, int hd, int splits,
                                           int early_trigger) {
  if (early_trigger) pdl_trigger();   // the next kernel is the o_proj GEMM
  pdl_wait();
  combine_head(part_ml, part_o, out, nh, hd, splits, blockIdx.y, blockIdx.x);
}

}  // namespace llama
