// bf16 projection / FFN GEMMs on the 5th-generation tensor cores (tcgen05).
//
// C = A · B^T with A [rows, K] and B [n, K] both K-major bf16, fp32
// accumulation in TMEM ([DeepDive] LLaMAAttention / LLaMAMLP: every Linear is
// y = x W^T with W [out, in]).  One CTA per SM, 10 warps:
//   warp 0      TMA producer (one elected lane): A and B tiles into a ring of
//               STAGES shared-memory stages, 128-byte swizzle, no multicast;
//   warp 1      TMEM allocator and MMA issuer (one lane): 4 x tcgen05.mma
//               (M=128, or 256 on a CTA pair; N=BN, K=16) per 64-wide
//               k-block, commit frees the stage;
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (one TMEM lane = one
//               output row per thread; two warps per lane quadrant, each
//               taking half of the tile's columns), fused epilogue, global
//               store.
// The accumulator is double-buffered in TMEM (2 x BN fp32 columns), so the
// epilogue of one tile overlaps the main loop of the next.
//
// Two schedules:
//  * tile mode (prefill, SWAP = false): A = activations (tokens x K),
//    B = weight rows.  A 2-CTA cluster (the two SMs of a TPC) computes one
//    256 x 256 tile with tcgen05 cta_group::2 MMAs (M = 256): each CTA loads
//    its 128 activation rows and half of the 256 weight rows per k-block and
//    holds its 128 x 256 half of the accumulator, so a CTA moves 32 KB instead
//    of 48 KB from L2 per k-block.  Persistent pairs walk the (m-tile, n-tile)
//    grid with the m index fastest inside groups of 8 m-tiles, so pairs that
//    run at the same time share weight tiles and at most 2048 activation rows
//    in L2.
//    Epilogues: bf16 store (QKV), QKV with RoPE and the KV-cache append
//    fused in (head_dim 64/128), fp32 residual add (o_proj, down; the
//    residual rows are prefetched into L2 during the tile's MMAs), paired
//    SiLU(gate)·up with the pair's B halves holding gate rows (rank 0) and the
//    matching up rows (rank 1) (gate_up), fp32 store (lm_head).
//  * stream-K mode (decode, SWAP = true): the weight is A (its rows fill the
//    MMA's M = 128) and the few token rows are B (N = BN >= tokens), so the
//    weight streams from HBM once.  The (weight tile, k-block) units are split
//    evenly over the CTAs and each CTA walks its range backwards: its only
//    piece that does not end a tile comes first and is published at once as
//    an fp32 partial plus a flag word; the CTA that holds a tile's last
//    k-block waits (bounded) for the lower CTAs' partials, adds them in CTA
//    order (deterministic) and applies the epilogue itself.  For gate_up a
//    weight tile is 64 gate rows followed by the matching 64 up rows, so
//    SiLU(gate)·up pairs TMEM lane r with lane r + 64 (through shared memory).
//    Cluster form (CL, at most 16 token rows, weight tiles <= SMs): one
//    thread-block cluster of S <= 8 CTAs per weight tile, each CTA taking
//    1/S of its k-blocks; ranks 1..S-1 store their fp32 pieces straight into
//    rank 0's shared memory (st.shared::cluster) and arrive on its mbarrier,
//    rank 0 adds them in rank order and applies the epilogue -- no L2 round
//    trip, flag word or wait on another cluster.
//
// The weight can be given as up to three row segments with their own tensor
// maps (q, k, v when the three projections are not contiguous; gate and up).
#pragma once

#include "common.cuh"

namespace llama {

// EPI_QKV_ROPE_BF16 (tile mode, head_dim 64 or 128): the QKV projection with
// RoPE and the KV-cache append fused in ([DeepDive] apply_rotary_emb; [MLX-13B]
// RoPE(traditional=True) and the cache concatenation): rotated q -> out,
// rotated k and v -> the cache at position p0 + t.
enum GemmEpi : int { EPI_BF16 = 0, EPI_RESID_F32 = 1, EPI_SWIGLU_BF16 = 2, EPI_F32 = 3, EPI_QKV_ROPE_BF16 = 4 };

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
  // EPI_QKV_ROPE_BF16: tokens m = b * L + t sit at position p0 + t
  void* kc;                // bf16 cache [batch][nkv][cap][hd]
  void* vc;
  const float* rope_tab;   // [M][hd]: cos of the token's hd/2 angles, then sin
  int L, p0, nh, nkv, hd, cap, rope_style;
  // stream-K mode
  float* partial;      // [grid][128 rows][BN tokens] fp32: each CTA's one non-final piece
  unsigned* flags;     // [grid]: 1 while that CTA's partial waits for its finisher, else 0
  long long units;     // n_tiles * num_kb
  DevStatus* status;
  unsigned long long limit_ns;
  // 1: signal dependents right after set-up, so the next kernel's CTAs launch
  // (and fetch their weights) while this one runs; 0: at the end of the work
  int early_trigger;
  // decode GEMM with the residual epilogue: the RMSNorm of the rows it
  // finishes, norm_out = bf16(norm_g * (out * rstd(out row))) (norm_g == nullptr: none)
  const float* norm_g;
  void* norm_out;
  float norm_eps;
  float* ssq;          // [n_tiles][BN]: per tile, the sum of squares of each token row's columns
  unsigned* norm_ctr;  // [2]: tiles finished, CTAs finished normalising (nullptr: ssq only)
  int sk_grid;         // stream-K: CTAs 0 .. sk_grid-1 share the units (<= gridDim.x, <= units)
  // cluster split (the CL kernel form): weight tile blockIdx.x / cl_split, its
  // k-blocks split over the cl_split CTAs of one thread-block cluster; ranks
  // 1.. store their fp32 pieces into rank 0's shared memory, which adds them
  int cl_split;
  // decode residual GEMM: write ssq (as with norm_g) for an RMSNorm done by the next GEMM
  int write_ssq;
  // cluster form only: the B operand (token rows) is RMSNorm(x) computed here
  // instead of loaded: bf16(nb_g * (x * rstd(x row))), rstd from the sums of
  // squares nb_ssq[tile][BN] of nb_tiles column tiles written by the GEMM
  // that produced x (nb_x == nullptr: B by TMA from the activation map)
  const float* nb_x;
  const float* nb_g;
  const float* nb_ssq;
  int nb_ldx, nb_tiles, nb_dim;
  float nb_eps;
  void* nb_h;          // bf16 [rows][nb_dim]: the normalised rows also stored here (by tile 0's cluster)
};

constexpr int GEMM_EPI_WARPS = 8;
constexpr int GEMM_THREADS = 64 + 32 * GEMM_EPI_WARPS;

// PAIR: tile mode on a CTA pair (M = 256 per MMA); this CTA holds 128 rows of
// A and BN / 2 rows of B per stage.  KS: 64-wide k sub-blocks per unit (decode:
// a stage then reads KS x 128 contiguous bytes of every weight row).
// CL: the cluster-split decode form (BN = 16), whose rank 0 also holds up to
// kMaxClusterSplit - 1 pieces of [128][BN] fp32.  Fewer stages make room, so
// that its shared memory stays within the plain form's: both then leave the
// SM the same L1 share for the kernel that follows under PDL (the CUDA-core
// decode attention streams the cache through L1).
constexpr int kMaxClusterSplit = 8;

template <int BN, bool PAIR, int KS = 1, bool CL = false>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_SUB = BM * BK * 2;
  static constexpr int B_SUB = (PAIR ? BN / 2 : BN) * BK * 2;
  static constexpr int A_BYTES = KS * A_SUB;
  static constexpr int B_BYTES = KS * B_SUB;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int CL_BYTES = CL ? (kMaxClusterSplit - 1) * 128 * BN * 4 : 0;
  static constexpr int STAGES_RAW = (200 * 1024) / STAGE_BYTES;
  static constexpr int STAGES_PLAIN = STAGES_RAW > 12 ? 12 : STAGES_RAW;
  static constexpr int STAGES = (STAGES_PLAIN * STAGE_BYTES - CL_BYTES) / STAGE_BYTES;
  static_assert(STAGES >= 2, "pipeline depth");
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                        : (2 * BN <= 256) ? 256 : 512;
  static constexpr int EXCH_BYTES = 2 * 64 * 16 * 4;   // gate/up pairing exchange (stream-K gate_up)
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256 + EXCH_BYTES + CL_BYTES;
};

// Work item shared by the three roles: one output tile and a k-block range.
struct GemmItem {
  int tile;   // tile mode: linear (m fastest); stream-K: weight tile
  int kb0, kb1;
};

struct GemmIter {
  // tile mode: one tile per CTA pair (cluster) at a time
  int next_tile, tile_count, tile_stride;
  // stream-K mode: this CTA's unit range [u0, u1), walked from the top
  long long u, u0;
  int num_kb;
  bool streamk;

  __device__ void init(const GemmParams& p, bool sk) {
    streamk = sk;
    num_kb = p.num_kb;
    if (!sk) {
      next_tile = blockIdx.x >> 1;
      tile_stride = gridDim.x >> 1;
      tile_count = p.m_tiles * p.n_tiles;
    } else if (p.cl_split > 0) {
      // one weight tile per cluster; this CTA's share of its k-blocks
      const long long S = p.cl_split, r = blockIdx.x % S, t = blockIdx.x / S;
      u0 = t * num_kb + num_kb * r / S;
      u = t * num_kb + num_kb * (r + 1) / S;
    } else {
      const long long G = p.sk_grid;
      if ((long long)blockIdx.x >= G) {
        u0 = u = 0;   // no share of this GEMM
      } else {
        u0 = p.units * (long long)blockIdx.x / G;
        u = p.units * (long long)(blockIdx.x + 1) / G;
      }
    }
  }
  __device__ bool next(GemmItem& it) {
    if (!streamk) {
      if (next_tile >= tile_count) return false;
      it.tile = next_tile;
      it.kb0 = 0;
      it.kb1 = num_kb;
      next_tile += tile_stride;
      return true;
    }
    if (u <= u0) return false;
    it.tile = (int)((u - 1) / num_kb);
    const long long start = (long long)it.tile * num_kb;
    const long long lo = u0 > start ? u0 : start;
    it.kb0 = (int)(lo - start);
    it.kb1 = (int)(u - start);
    u = lo;
    return true;
  }
};

// Tile mode: tile index -> (m-tile, weight tile); m runs fastest inside
// groups of up to 8 m-tiles (the last group may be smaller).
__device__ __forceinline__ void tile_coords(const GemmParams& p, int tile, int& mt, int& wt) {
  constexpr int GM = 8;
  const int per_group = GM * p.n_tiles;
  const int g = tile / per_group;
  const int gm = min(GM, p.m_tiles - g * GM);
  const int r = tile - g * per_group;
  wt = r / gm;
  mt = g * GM + r % gm;
}

__device__ __forceinline__ int seg_of_tile(const GemmParams& p, int wtile) {
  int s = 0;
  if (p.nseg > 1 && wtile >= p.seg_tile0[1]) s = 1;
  if (p.nseg > 2 && wtile >= p.seg_tile0[2]) s = 2;
  return s;
}

// mbarrier wait whose acquire covers writes that other CTAs of the cluster
// released into this CTA's shared memory before arriving.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Stream-K epilogue of one work item (decode form): the accumulator holds
// TMEM lane `row` = weight row of the tile, column j = token j.  A piece that
// does not end its tile is published for the tile's finisher; the CTA that
// ends the tile adds the pieces of the lower CTAs that share it, in CTA order,
// and applies the epilogue.  Called by every epilogue thread; `leader` is one
// of them (it handles the flag words), `xch` this thread's half of the
// gate/up exchange buffer in shared memory.
template <int BN, int EPI, typename Sync, bool CL = false>
__device__ __forceinline__ void streamk_epilogue(const GemmParams& p, const GemmItem& item, uint32_t tbase, int row,
                                                 int half, float* xch, bool leader, int* abort_sh, Sync& epi_sync,
                                                 float (*red)[16], float* cl_buf = nullptr, uint32_t red_bar = 0) {
  // accumulator: TMEM lane `row` = weight row of the tile, column j = token j
  const uint32_t cl_rank = CL ? blockIdx.x % (unsigned)p.cl_split : 0u;
  if (CL && cl_rank > 0) {
    // a piece of the cluster's tile: into slot rank - 1 of rank 0's shared memory
    const uint32_t dst = mapa_shared(smem_u32(cl_buf + ((size_t)(cl_rank - 1) * 128 + row) * BN), 0);
#pragma unroll 1
    for (int c = half * 16; c < BN; c += 32) {
      float v[16];
      tmem_ld16(tbase + c, v);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q)
        asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst + (uint32_t)(c + 4 * q) * 4u),
                     "f"(v[4 * q]), "f"(v[4 * q + 1]), "f"(v[4 * q + 2]), "f"(v[4 * q + 3])
                     : "memory");
    }
    epi_sync();
    if (leader) {
      asm volatile("fence.acq_rel.cluster;" ::: "memory");
      mbar_arrive_remote(mapa_shared(red_bar, 0));
    }
    return;
  }
  if (!CL && item.kb1 < p.num_kb) {
    // a piece that does not end its tile: publish it for the tile's finisher
    float* dst = p.partial + ((size_t)blockIdx.x * 128 + row) * BN;
#pragma unroll 1
    for (int c = half * 16; c < BN; c += 32) {
      float v[16];
      tmem_ld16(tbase + c, v);
      tmem_ld_wait();
      float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
      for (int q = 0; q < 4; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
    // the group barrier orders every thread's stores before thread 64's
    // release, which makes them visible at GPU scope before the flag
    epi_sync();
    if (leader)
      asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p.flags + blockIdx.x), "r"(1u) : "memory");
  } else {
    // this CTA ends the tile: add the partials of the lower CTAs that share it
    const unsigned U = (unsigned)p.units, G = (unsigned)p.sk_grid, KB = (unsigned)p.num_kb;
    const unsigned x = (unsigned)item.tile * KB;
    int c_first = (int)(((x + 1) * G + U - 1) / U) - 1;
    c_first = c_first < 0 ? 0 : c_first;
    // CTAs c_first .. blockIdx.x-1 (none has an empty range: the grid is at most the unit count);
    // cluster split: ranks 1 .. cl_split - 1, from this CTA's shared memory
    const int n_contrib = CL ? p.cl_split - 1 : (int)blockIdx.x - c_first;
    if (CL && n_contrib > 0) {
      if (leader) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_cluster(red_bar, 0)) {
          if (*reinterpret_cast<volatile int*>(abort_sh)) break;
          if (globaltimer_ns() - t0 > p.limit_ns) {
            *abort_sh = 1;
            record_error(p.status, LLAMA_ERR_DEVICE_TIMEOUT, 14, item.tile);
            break;
          }
        }
      }
      epi_sync();
    } else if (n_contrib > 0) {
      // the first epilogue warp waits for the contributors' flags, one lane
      // each, so the waits overlap (one L2 round trip instead of one per piece)
      if ((threadIdx.x >> 5) == 2) {
        const int lane = (int)(threadIdx.x & 31);
        const uint64_t t0 = globaltimer_ns();
        for (int c = c_first + lane; c < (int)blockIdx.x; c += 32) {
          while (true) {
            unsigned f;
            asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(f) : "l"(p.flags + c) : "memory");
            if (f == 1u || *reinterpret_cast<volatile int*>(abort_sh)) break;
            if (globaltimer_ns() - t0 > p.limit_ns) {
              *abort_sh = 1;
              record_error(p.status, LLAMA_ERR_DEVICE_TIMEOUT, 6, item.tile);
              break;
            }
            __nanosleep(32);
          }
          // this CTA is the only reader of c's piece: re-arm the flag for the next launch
          asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p.flags + c), "r"(0u) : "memory");
        }
        asm volatile("fence.acq_rel.gpu;" ::: "memory");   // the pieces are read after the flags were seen
        __syncwarp();
      }
      epi_sync();
    }
    // weight row -> output column
    int seg = 0, n = 0;
    bool n_ok;
    if (EPI == EPI_SWIGLU_BF16) {
      n = item.tile * 64 + (row & 63);
      n_ok = n < p.seg_rows[0];
    } else {
      seg = seg_of_tile(p, item.tile);
      const int r_in_seg = (item.tile - p.seg_tile0[seg]) * 128 + row;
      n_ok = r_in_seg < p.seg_rows[seg];
      n = p.seg_col0[seg] + r_in_seg;
    }
  #pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 32) {
      const int c = c0 + half * 16;   // this warp's 16 token columns (BN is a multiple of 16)
      const bool active = c < BN;
      float v[16];
      if (active) {
        tmem_ld16(tbase + c, v);
        tmem_ld_wait();
        // the contributors' pieces, in CTA (rank) order, up to four per round trip
        const float4* src = reinterpret_cast<const float4*>(
            CL ? cl_buf + (size_t)row * BN + c : p.partial + ((size_t)c_first * 128 + row) * BN + c);
        constexpr size_t STRIDE4 = (size_t)128 * BN / 4;
#pragma unroll 1
        for (int k = 0; k < n_contrib; k += 4) {
          float4 a[4][4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              a[i][q] = k + i < n_contrib ? (CL ? src[(size_t)(k + i) * STRIDE4 + q]
                                                : __ldcg(src + (size_t)(k + i) * STRIDE4 + q))
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              v[4 * q + 0] += a[i][q].x;
              v[4 * q + 1] += a[i][q].y;
              v[4 * q + 2] += a[i][q].z;
              v[4 * q + 3] += a[i][q].w;
            }
        }
      }
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
            if (c + j < p.act_rows)
              o[(size_t)(c + j) * p.ldo + n] = __float2bfloat16_rn(silu_f(v[j]) * xch[j * 64 + row]);
        }
        epi_sync();
      } else {
        float xo[16];   // the outputs this thread writes (zero elsewhere), for a fused RMSNorm
#pragma unroll
        for (int j = 0; j < 16; ++j) xo[j] = 0.f;
        const int nj = p.act_rows - c < 16 ? p.act_rows - c : 16;
        if (EPI == EPI_RESID_F32 && active && n_ok) {
          // all residual loads first (out may alias resid: same element, same thread)
          float r[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) r[j] = j < nj ? __ldcg(p.resid + (size_t)(c + j) * p.ldr + n) : 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < nj) {
              xo[j] = r[j] + v[j];
              reinterpret_cast<float*>(p.out)[(size_t)(c + j) * p.ldo + n] = xo[j];
            }
        } else if (active && n_ok) {
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
        if (EPI == EPI_RESID_F32 && (p.norm_g != nullptr || p.write_ssq)) {
          // this tile's share of each token row's sum of squares: over the warp's
          // 32 rows by a halving butterfly (each step a lane keeps half of its
          // 16 sums and adds its partner's copy of them: 16 shuffles, after
          // which lanes 2j and 2j + 1 hold token j's sum), then over the four
          // warps of the same column half
          const int ew = (int)(threadIdx.x >> 5) - 2, lane = (int)(threadIdx.x & 31);
          float sq[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) sq[j] = xo[j] * xo[j];
#pragma unroll
          for (int st = 0; st < 4; ++st) {
            const int W = 8 >> st, bit = 16 >> st;
            const bool upper = (lane & bit) != 0;
#pragma unroll
            for (int i = 0; i < W; ++i) {
              const float send = upper ? sq[i] : sq[i + W];
              const float keep = upper ? sq[i + W] : sq[i];
              sq[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
            }
          }
          sq[0] += __shfl_xor_sync(0xffffffffu, sq[0], 1);
          if ((lane & 1) == 0) red[ew][lane >> 1] = sq[0];
          epi_sync();
          const int e = (int)threadIdx.x - 64;
          if (e < 32) {
            const int hh = e >> 4, j = e & 15, c2 = c0 + 16 * hh + j;
            if (c2 < BN) {
              float q = 0.f;
#pragma unroll
              for (int w = 0; w < 4; ++w) q += red[4 * hh + w][j];
              p.ssq[(size_t)item.tile * BN + c2] = q;
            }
          }
          // red is reused by the next column block or work item, and the fused
          // RMSNorm counts the tile after this barrier; a cluster-form CTA's
          // last block with the sums only has neither
          if (!(CL && p.norm_g == nullptr && c0 + 32 >= BN)) epi_sync();
        }
      }
    }
    if (EPI == EPI_RESID_F32 && p.norm_g != nullptr && p.norm_ctr != nullptr && leader) {
      // the tile's outputs and sums are written (ordered by the group barriers): count it
      asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p.norm_ctr), "r"(1u) : "memory");
    }
  }
}

// RMSNorm of the rows a decode residual GEMM finished ([MLX-13B] 4. RMSNorm;
// [DeepDive] LLaMARMSNorm), run by the epilogue threads of every CTA once
// their own tiles are done: wait (bounded) until every tile is counted, rstd
// of each token row from the tiles' sums of squares, then this CTA's share of
// the columns, h = g * (x * rstd).  The last CTA re-arms the counters.
template <int BN, typename Sync>
__device__ __forceinline__ void fused_rmsnorm(const GemmParams& p, bool leader, int* abort_sh, Sync& epi_sync,
                                              float* rstd_sh) {
  if (leader) {
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      unsigned f;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(f) : "l"(p.norm_ctr) : "memory");
      if (f >= (unsigned)p.n_tiles || *reinterpret_cast<volatile int*>(abort_sh)) break;
      if (globaltimer_ns() - t0 > p.limit_ns) {
        *abort_sh = 1;
        record_error(p.status, LLAMA_ERR_DEVICE_TIMEOUT, 11, 0);
        break;
      }
      __nanosleep(64);
    }
  }
  epi_sync();
  const int e = (int)threadIdx.x - 64;
  const int dim = p.seg_rows[0];
  const bool ok = *reinterpret_cast<volatile int*>(abort_sh) == 0;
  if (ok) {
    for (int j = e; j < p.act_rows; j += 32 * GEMM_EPI_WARPS) {
      float q = 0.f;
      for (int t = 0; t < p.n_tiles; ++t) q += __ldcg(p.ssq + (size_t)t * BN + j);
      rstd_sh[j] = rsqrtf(q / (float)dim + p.norm_eps);
    }
  }
  epi_sync();
  if (ok) {
    const int n0 = (int)((long long)dim * blockIdx.x / gridDim.x);
    const int n1 = (int)((long long)dim * (blockIdx.x + 1) / gridDim.x);
    const int w = n1 - n0;
    const float* x = reinterpret_cast<const float*>(p.out);
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(p.norm_out);
    for (int i = e; i < w * p.act_rows; i += 32 * GEMM_EPI_WARPS) {
      const int j = i / w, n = n0 + i % w;
      h[(size_t)j * dim + n] = __float2bfloat16_rn(__ldg(p.norm_g + n) * (__ldcg(x + (size_t)j * p.ldo + n) * rstd_sh[j]));
    }
  }
  epi_sync();
  if (leader) {
    __threadfence();
    if (atomicAdd(p.norm_ctr + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.norm_ctr, 0u);
      atomicExch(p.norm_ctr + 1, 0u);
    }
  }
}

template <int BN, bool SWAP, int EPI, int KS = 1, bool CL = false>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmAct, const __grid_constant__ CUtensorMap tmW0,
                   const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2,
                   const GemmParams p) {
  constexpr bool PAIR = !SWAP;            // tile mode runs 256 x BN tiles on CTA pairs
  static_assert(KS == 1 || SWAP, "k sub-blocks are a decode (stream-K) form");
  static_assert(!CL || (SWAP && BN == 16 && KS == 2), "the cluster split is a decode form of 16 token columns");
  using C = GemmCfg<BN, PAIR, KS, CL>;
  constexpr int STAGES = C::STAGES;
  constexpr int WROWS = SWAP ? 128 : BN;  // weight rows per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain, epilogue group, cluster pieces
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float red_sh[SWAP ? GEMM_EPI_WARPS : 1][16];   // fused RMSNorm: per-warp sums
  __shared__ float rstd_sh[SWAP ? 128 : 1];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;   // 0: issues the pair's MMAs
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  const uint32_t epi_bar = bar0 + 8u * (2 * STAGES + 5);
  const uint32_t red_bar = bar0 + 8u * (2 * STAGES + 6);
  // cluster form with the RMSNorm in the prologue: the epilogue threads write B
  const bool norm_b = CL && p.nb_x != nullptr;
  static_assert(8 * (2 * STAGES + 7) <= 256, "barrier block");
  // cluster split: the other ranks' pieces, in rank 0's shared memory
  float* cl_buf = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES + 256 + C::EXCH_BYTES);

  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < STAGES; ++s) {
      // (+ one arrival per epilogue thread when they write the B operand)
      mbar_init(full_bar(s), norm_b ? 1 + 32 * GEMM_EPI_WARPS : 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      // pair: one arrival per epilogue warp of both CTAs (on rank 0's barrier)
      mbar_init(acce_bar(b), PAIR ? 2 * GEMM_EPI_WARPS : 32 * GEMM_EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    mbar_init(epi_bar, 32 * GEMM_EPI_WARPS);
    if (CL) mbar_init(red_bar, p.cl_split > 1 ? p.cl_split - 1 : 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if (!norm_b) tma_prefetch_desc(&tmAct);
    tma_prefetch_desc(&tmW0);
    if (p.nseg > 1) tma_prefetch_desc(&tmW1);
    if (p.nseg > 2) tma_prefetch_desc(&tmW2);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(&tmem_base_sh), C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&tmem_base_sh), C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  // pair: the peer's TMA loads and the leader's commits target barriers of the
  // other CTA, so both must be initialised before either proceeds (cluster
  // split: the other ranks arrive on rank 0's red_bar)
  if constexpr (PAIR || CL) cluster_sync(); else __syncthreads();
  tc_fence_after();
  if (p.early_trigger) pdl_trigger();
  // stream-K (decode): the producer starts the weight stream before its PDL wait
  if (!(SWAP && warp == 0)) pdl_wait();
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
      // weight tile of unit kb (KS sub-blocks of 64) of weight tile wtile (stream-K mode) into A stage sa
      auto load_weight_swap = [&](uint32_t sa, uint32_t bar, int wtile, int kb) {
#pragma unroll
        for (int i = 0; i < KS; ++i) {
          const int x = (kb * KS + i) * 64;
          const uint32_t dst = sa + i * C::A_SUB;
          if (EPI == EPI_SWIGLU_BF16) {
            // 64 gate rows into lanes 0..63 of the tile, the same 64 up rows into 64..127
            tma_load_2d(dst, &tmW0, bar, x, wtile * 64);
            tma_load_2d(dst + 64 * 128, &tmW1, bar, x, wtile * 64);
          } else {
            const int seg = seg_of_tile(p, wtile);
            const CUtensorMap* wm = seg == 0 ? &tmW0 : (seg == 1 ? &tmW1 : &tmW2);
            tma_load_2d(dst, wm, bar, x, (wtile - p.seg_tile0[seg]) * 128);
          }
        }
      };
      auto load_act_swap = [&](uint32_t sb, uint32_t bar, int kb) {
#pragma unroll
        for (int i = 0; i < KS; ++i) tma_load_2d(sb + i * C::B_SUB, &tmAct, bar, (kb * KS + i) * 64, 0);
      };
      int skip = 0;   // k-blocks already issued before the PDL wait
      if (SWAP) {
        // The weights do not depend on the previous kernel: fill every stage's
        // weight tile first, wait for the previous kernel, then add the
        // activation tiles.  Every stage is empty at this point.
        int pre_kb[STAGES];
        GemmIter it;
        it.init(p, true);
        GemmItem item;
        while (skip < STAGES && it.next(item)) {
          for (int kb = item.kb0; kb < item.kb1 && skip < STAGES; ++kb) {
            mbar_arrive_expect_tx(full_bar(skip), norm_b ? C::A_BYTES : C::STAGE_BYTES);
            load_weight_swap(smem_u32(smem + skip * C::STAGE_BYTES), full_bar(skip), item.tile, kb);
            pre_kb[skip++] = kb;
          }
        }
        pdl_wait();
        for (int s = 0; s < skip; ++s) {
          if (!norm_b) load_act_swap(smem_u32(smem + s * C::STAGE_BYTES) + C::A_BYTES, full_bar(s), pre_kb[s]);
          filled_parity[s] = 0;
        }
        stage = skip % STAGES;
        phase = skip == STAGES ? 1u : 0u;
      }
      GemmIter it;
      it.init(p, SWAP);
      GemmItem item;
      bool ok = true;
      while (ok && it.next(item)) {
        int wtile, m0 = 0;
        if (SWAP) {
          wtile = item.tile;
        } else {
          int mt;
          tile_coords(p, item.tile, mt, wtile);
          m0 = mt * 256 + 128 * (int)rank;
        }
        const int seg = seg_of_tile(p, wtile);
        const int wrow0 = (wtile - p.seg_tile0[seg]) * WROWS + (PAIR ? (BN / 2) * (int)rank : 0);
        const CUtensorMap* wm = seg == 0 ? &tmW0 : (seg == 1 ? &tmW1 : &tmW2);
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
          const uint32_t sb = sa + C::A_BYTES;
          if (SWAP) {
            mbar_arrive_expect_tx(full_bar(stage), norm_b ? C::A_BYTES : C::STAGE_BYTES);
            load_weight_swap(sa, full_bar(stage), wtile, kb);
            if (!norm_b) load_act_swap(sb, full_bar(stage), kb);
          } else {
            // both CTAs' bytes land on rank 0's full barrier, which rank 0 arms
            if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * C::STAGE_BYTES);
            const uint32_t lbar = mapa_shared(full_bar(stage), 0);
            tma_load_2d_pair(sa, &tmAct, lbar, kb * 64, m0);
            if (EPI == EPI_SWIGLU_BF16) {
              // B columns 0..BN/2-1 (rank 0) are gate rows, BN/2..BN-1 (rank 1) the matching up rows
              tma_load_2d_pair(sb, rank == 0 ? &tmW0 : &tmW1, lbar, kb * 64, wtile * (BN / 2));
            } else {
              tma_load_2d_pair(sb, wm, lbar, kb * 64, wrow0);
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
      // (pair: rank 0's full barriers count both CTAs' loads; rank 1 leaves
      // only after the closing cluster barrier, which rank 0 reaches after this)
      if (!PAIR || rank == 0)
        for (int s = 0; s < STAGES; ++s)
          if (filled_parity[s] >= 0) mbar_wait(full_bar(s), (uint32_t)filled_parity[s], wc, 9, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(PAIR ? 256 : 128, BN, 0, 0);
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
          for (int i = 0; i < KS; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t ad = smem_desc_sw128(sa + i * C::A_SUB + k * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(sb + i * C::B_SUB + k * 32, 16, 1024);
              const uint32_t acc = (kb > item.kb0 || i > 0 || k > 0) ? 1u : 0u;
              if constexpr (PAIR)
                umma_bf16_pair(d_tmem, ad, bd, IDESC, acc);
              else
                umma_bf16(d_tmem, ad, bd, IDESC, acc);
            }
          issued = true;
          if constexpr (PAIR) umma_commit_pair(empty_bar(stage), 3); else umma_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (PAIR) umma_commit_pair(accf_bar(abuf), 3); else umma_commit(accf_bar(abuf));
        if (++abuf == 2) {
          abuf = 0;
          aphase ^= 1u;
        }
      }
      if constexpr (PAIR) {
        // always (also with nothing issued): rank 1 waits on its copy before
        // it releases TMEM and leaves
        umma_commit_pair(drain_bar, 3);
        mbar_wait(drain_bar, 0, wc, 8, false);
      } else if (issued) {
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
    // Barrier of the epilogue warps: an mbarrier with a bounded wait rather than
    // a named barrier, so a warp that left the loop on an error cannot hang the rest.
    uint32_t epi_phase = 0;
    auto epi_sync = [&]() {
      mbar_arrive(epi_bar);
      mbar_wait(epi_bar, epi_phase, wc, 7);
      epi_phase ^= 1u;
    };
    if constexpr (CL) {
      if (norm_b) {
        // B operand = RMSNorm of the token rows ([MLX-13B] 4. RMSNorm;
        // [DeepDive] LLaMARMSNorm), written into each stage as TMA would lay
        // it out (128-byte rows, 16-byte chunk c of row r at c ^ (r & 7)):
        // thread e takes token row e / 16 and 8 consecutive k of each k-block.
        const int e = (int)threadIdx.x - 64;
        static_assert(BN * 16 == 32 * GEMM_EPI_WARPS, "one 16-byte chunk per thread and k-block");
        const int brow = e >> 4, sub = (e >> 3) & 1, chunk = e & 7;
        const bool brow_ok = brow < p.act_rows;
        const uint32_t boff = (uint32_t)(C::A_BYTES + sub * C::B_SUB + brow * 128 + ((chunk ^ (brow & 7)) << 4));
        // the first weight tile's cluster covers every k once: it also stores the rows
        const bool store_h = p.nb_h != nullptr && (int)blockIdx.x < p.cl_split;
        GemmIter bit;
        bit.init(p, true);
        GemmItem bitem;
        const bool have = bit.next(bitem);   // the cluster form gives a CTA one item
        const int kbeg = have ? bitem.kb0 : 0, kend = have ? bitem.kb1 : 0;
        // this thread's x and g for a k-block, three k-blocks ahead of the stores
        constexpr int AHEAD = 3;
        float4 xq[AHEAD][2], gq[AHEAD][2];
        auto fetch = [&](int kb, float4 (&xs)[2], float4 (&gs)[2]) {
          const int k0 = (kb * KS + sub) * 64 + chunk * 8;
          if (kb < kend && brow_ok && k0 < p.K) {
            const float4* xr = reinterpret_cast<const float4*>(p.nb_x + (size_t)brow * p.nb_ldx + k0);
            const float4* gr = reinterpret_cast<const float4*>(p.nb_g + k0);
            xs[0] = __ldcg(xr);
            xs[1] = __ldcg(xr + 1);
            gs[0] = __ldg(gr);
            gs[1] = __ldg(gr + 1);
          } else {
            xs[0] = xs[1] = gs[0] = gs[1] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        };
#pragma unroll
        for (int a = 0; a < AHEAD; ++a) fetch(kbeg + a, xq[a], gq[a]);
        // rstd of each token row from the producing GEMM's per-tile sums of
        // squares: 16 threads per row (lanes of one half-warp) split the tiles
        {
          const int r = e >> 4, part = e & 15;
          float ss = 0.f;
          for (int t = part; t < p.nb_tiles; t += 16) ss += __ldcg(p.nb_ssq + (size_t)t * BN + r);
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          if (part == 0) rstd_sh[r] = rsqrtf(ss / (float)p.nb_dim + p.nb_eps);
        }
        epi_sync();
        const float rs = rstd_sh[brow];
        for (int n = 0; n < kend - kbeg; ++n) {
          const int kb = kbeg + n, stage = n % STAGES;
          if (!mbar_wait(empty_bar(stage), ((uint32_t)(n / STAGES) & 1u) ^ 1u, wc, 13)) break;
          const int k0 = (kb * KS + sub) * 64 + chunk * 8;
          uint4 o;
          o.x = pack_bf16x2(gq[0][0].x * (xq[0][0].x * rs), gq[0][0].y * (xq[0][0].y * rs));
          o.y = pack_bf16x2(gq[0][0].z * (xq[0][0].z * rs), gq[0][0].w * (xq[0][0].w * rs));
          o.z = pack_bf16x2(gq[0][1].x * (xq[0][1].x * rs), gq[0][1].y * (xq[0][1].y * rs));
          o.w = pack_bf16x2(gq[0][1].z * (xq[0][1].z * rs), gq[0][1].w * (xq[0][1].w * rs));
          if (store_h && brow_ok && k0 < p.K)
            *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.nb_h) + (size_t)brow * p.nb_dim + k0) = o;
          const uint32_t dst = smem_u32(smem + stage * C::STAGE_BYTES) + boff;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(o.x), "r"(o.y), "r"(o.z), "r"(o.w)
                       : "memory");
          // generic-proxy writes, read by the tensor core through the async proxy
          // (one arrival per thread: measured faster than a warp sync and one
          // arrival per warp)
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          mbar_arrive(full_bar(stage));
#pragma unroll
          for (int a = 0; a + 1 < AHEAD; ++a) {
            xq[a][0] = xq[a + 1][0];
            xq[a][1] = xq[a + 1][1];
            gq[a][0] = gq[a + 1][0];
            gq[a][1] = gq[a + 1][1];
          }
          fetch(kb + AHEAD, xq[AHEAD - 1], gq[AHEAD - 1]);
        }
      }
    }
    int abuf = 0;
    uint32_t aphase = 0;
    GemmIter it;
    it.init(p, SWAP);
    GemmItem item;
    while (it.next(item)) {
      if constexpr (PAIR && EPI == EPI_RESID_F32) {
        // While this tile's MMAs run, pull this thread's residual row segment
        // (half of the tile's columns, 4 x 128 B of fp32) into L2, so that the
        // epilogue -- exposed for a CTA's last tile -- does not wait on DRAM.
        int mt, wt;
        tile_coords(p, item.tile, mt, wt);
        const int m = mt * 256 + 128 * (int)rank + row;
        const int sg = seg_of_tile(p, wt);
        const int nl = (wt - p.seg_tile0[sg]) * BN + half * (BN / 2);
        if (m < p.act_rows && nl < p.seg_rows[sg]) {
          const float* r = p.resid + (size_t)m * p.ldr + p.seg_col0[sg] + nl;
#pragma unroll
          for (int q = 0; q < BN / 64; ++q)
            if (nl + 32 * q < p.seg_rows[sg]) asm volatile("prefetch.global.L2 [%0];" ::"l"(r + 32 * q));
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(accf_bar(abuf), aphase, wc, 4))) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(abuf * BN);
      if constexpr (SWAP) {
        streamk_epilogue<BN, EPI, decltype(epi_sync), CL>(
            p, item, tbase, row, half,
            reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES + 256) + half * (64 * 16), threadIdx.x == 64,
            &abort_sh, epi_sync, red_sh, cl_buf, red_bar);
      } else {
        int mt, wtile;
        tile_coords(p, item.tile, mt, wtile);
        const int m = mt * 256 + 128 * (int)rank + row;
        const bool row_ok = m < p.act_rows;

        if constexpr (EPI == EPI_QKV_ROPE_BF16) {
          const int seg = seg_of_tile(p, wtile);
          const int nl0 = (wtile - p.seg_tile0[seg]) * BN + half * (BN / 2);   // this warp's first row in the segment
          const int nlim = p.seg_rows[seg];
          const int n0 = p.seg_col0[seg] + nl0;                                // its first qkv column
          const int hd = p.hd, nq = p.nh * hd, nk = p.nkv * hd;
          const int bseq = row_ok ? m / p.L : 0;
          const int pos = p.p0 + (m - bseq * p.L);
          const bool halfstyle = p.rope_style == 0;
          // this token's angles, computed once per token by the first RMSNorm
          const float* cst = p.rope_tab + (size_t)(row_ok ? m : 0) * hd;
          const float* snt = cst + hd / 2;
          auto load16 = [](const float* src, float* dst) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 t = __ldg(reinterpret_cast<const float4*>(src) + q);
              dst[4 * q] = t.x;
              dst[4 * q + 1] = t.y;
              dst[4 * q + 2] = t.z;
              dst[4 * q + 3] = t.w;
            }
          };
          auto rot = [](float c, float s, float& x0, float& x1) {
            const float y0 = x0 * c - x1 * s, y1 = x1 * c + x0 * s;
            x0 = y0;
            x1 = y1;
          };
          // destination of the 32 columns starting at qkv column n (inside one head)
          auto dst = [&](int n) -> __nv_bfloat16* {
            if (n < nq) return reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)m * p.ldo + n;
            const bool is_k = n < nq + nk;
            const int r = is_k ? n - nq : n - nq - nk;
            __nv_bfloat16* c = reinterpret_cast<__nv_bfloat16*>(is_k ? p.kc : p.vc);
            return c + (((size_t)bseq * p.nkv + r / hd) * p.cap + pos) * hd + r % hd;
          };
          auto store32 = [&](__nv_bfloat16* o, const float (&v)[32]) {
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
          };
          // Two passes over two 32-column chunks (a, b) of this warp's 128 columns.
          // Rotate-half pairs column d with d + hd/2: hd 128 -> (0, 64), (32, 96);
          // hd 64 -> (0, 32), (64, 96).  Interleaved pairs and v stay in a chunk.
#pragma unroll 1
          for (int pass = 0; pass < 2; ++pass) {
            const int ca = (halfstyle && hd == 128) ? 32 * pass : 64 * pass;
            const int cb = (halfstyle && hd == 128) ? ca + 64 : ca + 32;
            float va[32], vb[32];
            tmem_ld32(tbase + half * (BN / 2) + ca, va);
            tmem_ld32(tbase + half * (BN / 2) + cb, vb);
            tmem_ld_wait();
            if (!row_ok || nl0 + ca >= nlim) continue;   // segments end on 32-column boundaries
            const int na = n0 + ca, nb = n0 + cb;
            const bool b_ok = nl0 + cb < nlim;
            if (na < nq + nk) {   // q or k: rotate
              const int da = na % hd;
              float cs[32], sn[32];
              if (halfstyle) {
                // pair i = da + j: (va[j], vb[j])
                load16(cst + da, cs);
                load16(cst + da + 16, cs + 16);
                load16(snt + da, sn);
                load16(snt + da + 16, sn + 16);
#pragma unroll
                for (int j = 0; j < 32; ++j) rot(cs[j], sn[j], va[j], vb[j]);
              } else {
                // pairs (2i, 2i+1) inside each chunk: i = da/2 + j and db/2 + j
                const int db = nb % hd;
                load16(cst + da / 2, cs);
                load16(cst + db / 2, cs + 16);
                load16(snt + da / 2, sn);
                load16(snt + db / 2, sn + 16);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  rot(cs[j], sn[j], va[2 * j], va[2 * j + 1]);
                  rot(cs[16 + j], sn[16 + j], vb[2 * j], vb[2 * j + 1]);
                }
              }
            }
            store32(dst(na), va);
            if (b_ok) store32(dst(nb), vb);
          }
        } else if (EPI == EPI_SWIGLU_BF16) {
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
      if constexpr (PAIR) {
        __syncwarp();   // every lane's TMEM reads are complete (waited above)
        if (lane == 0) mbar_arrive_remote(mapa_shared(acce_bar(abuf), 0));
      } else {
        mbar_arrive(acce_bar(abuf));
      }
      if (++abuf == 2) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
    if constexpr (SWAP && EPI == EPI_RESID_F32)
      if (p.norm_g != nullptr) fused_rmsnorm<BN>(p, threadIdx.x == 64, &abort_sh, epi_sync, rstd_sh);
  }

  pdl_trigger();   // the next kernel may start its prologue while this CTA tears down
  tc_fence_before();
  // pair: neither CTA leaves while the other may still use its shared memory
  // (rank 0's MMAs read rank 1's stages; rank 1's epilogue arrives on rank 0);
  // cluster split: rank 0 stays while the others may still store their pieces
  if constexpr (PAIR || CL) cluster_sync(); else __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    if constexpr (PAIR) {
      // rank 0's MMAs also wrote this CTA's TMEM
      bool drained = true;
      if (lane == 0) drained = mbar_wait(drain_bar, 0, wc, 8, false);
      (void)drained;
      __syncwarp();
      tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    } else {
      tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
  }
}

}  // namespace llama
