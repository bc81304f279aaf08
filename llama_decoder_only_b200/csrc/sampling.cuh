// Temperature / top-p (nucleus) sampling of the next token from the
// lm_head's logits ([DeepDive] class LLaMA, generate: logits / temperature,
// sort descending, cumulative softmax, drop a token once the probability
// sorted before it exceeds top_p, renormalise, draw; [MLX-13B] 生成过程:
// temperature 0 is greedy argmax).
//
// The draw is an input: one uniform u in [0, 1) per sequence, and the token
// is the one whose interval of the cumulative renormalised distribution
// (in sorted order) holds u.  Sorted order is descending logit, ties by
// ascending vocabulary index.
//
// No sort is materialised.  Each token gets a unique 64-bit key whose
// descending order is the sorted order (order-preserving bits of z = logit /
// temperature, then the complemented index), and an integer mass
// w = round(2^40 exp(z - max z)) -- integers, so every sum is exact and the
// result does not depend on the order of the additions.  "The token whose
// cumulative interval [before, before + w) holds a target" is found by a
// radix walk over the key from its top byte down: per pass, a 256-bin
// histogram of the masses of the tokens still in play, a scan from the top
// bin to the one that holds the target, and the mass above it carried on.
// The walk runs twice: the top-p cut (target top_p * W; the token found is
// the last one kept, so the kept mass is its before + w) and the draw
// (target u * kept mass).  One CTA per sequence; logits are read from global
// memory (L2) on each pass.
#pragma once

#include "common.cuh"

namespace llama {

constexpr int SAMPLE_THREADS = 1024;

__device__ __forceinline__ uint32_t desc_key_f32(float z) {
  const uint32_t u = __float_as_uint(z);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);   // larger z -> larger key
}

struct SampleShared {
  unsigned long long hist[256];
  unsigned int cnt[256];
  unsigned long long wsum;
  float red_f[32];
  unsigned long long red_u[32];
  unsigned long long sel_prefix, sel_mask, sel_above, sel_w;
  int sel_done;
};

// Mass of token i: exp(z_i - zmax) in fp32, as an integer in units of 2^-40.
__device__ __forceinline__ unsigned long long token_mass(float z, float zmax) {
  const float e = expf(z - zmax);                      // in (0, 1]
  return __float2ull_rn(e * 1099511627776.0f);         // 2^40
}

__device__ __forceinline__ unsigned long long token_key(float z, int i) {
  return ((unsigned long long)desc_key_f32(z) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)i);
}

// Radix walk: the token whose interval [before, before + w) of the
// cumulative mass in descending key order holds `target` (< total mass).
// Returns (through shared memory) its key's bits, the mass before it and its
// own mass.  All threads of the CTA call it.
__device__ void select_by_mass(const float* __restrict__ row, int V, float temp, float zmax,
                               unsigned long long target, SampleShared& sh) {
  if (threadIdx.x == 0) {
    sh.sel_prefix = 0;
    sh.sel_mask = 0;
    sh.sel_above = 0;
    sh.sel_done = 0;
  }
  __syncthreads();
#pragma unroll 1
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
      sh.hist[b] = 0;
      sh.cnt[b] = 0;
    }
    __syncthreads();
    const unsigned long long prefix = sh.sel_prefix, mask = sh.sel_mask;
    for (int i = threadIdx.x; i < V; i += blockDim.x) {
      const float z = row[i] / temp;
      const unsigned long long k = token_key(z, i);
      if ((k & mask) == prefix) {
        const int b = (int)((k >> shift) & 255u);
        atomicAdd(&sh.hist[b], token_mass(z, zmax));
        atomicAdd(&sh.cnt[b], 1u);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      // from the top bin down: the first bin whose upper edge passes the target
      unsigned long long above = sh.sel_above;
      int bsel = -1;
      for (int b = 255; b >= 0; --b) {
        if (sh.cnt[b] == 0) continue;
        if (target < above + sh.hist[b]) {
          bsel = b;
          break;
        }
        above += sh.hist[b];
      }
      if (bsel < 0) {
        // rounding left the target at the very end: take the last token in play
        for (int b = 0; b < 256; ++b)
          if (sh.cnt[b] != 0) {
            bsel = b;
            break;
          }
        above = sh.sel_above;
        for (int b = 255; b > bsel; --b) above += sh.hist[b];
      }
      sh.sel_prefix = prefix | ((unsigned long long)bsel << shift);
      sh.sel_mask = mask | (255ull << shift);
      sh.sel_above = above;
      sh.sel_w = sh.hist[bsel];
      sh.sel_done = sh.cnt[bsel] == 1;
    }
    __syncthreads();
    if (sh.sel_done) break;
  }
  // with one token left in the chosen bin, its full key comes from one more pass
  if (sh.sel_done) {
    const unsigned long long prefix = sh.sel_prefix, mask = sh.sel_mask;
    for (int i = threadIdx.x; i < V; i += blockDim.x) {
      const unsigned long long k = token_key(row[i] / temp, i);
      if ((k & mask) == prefix) sh.sel_prefix = k;   // exactly one writer
    }
    __syncthreads();
  }
}

// ids[b] for logits [B, V] (row b at logits + b * V); u [B] device uniforms.
// temperature > 0 (temperature 0 is served by the argmax kernel); top_p in (0, 1].
__global__ void __launch_bounds__(SAMPLE_THREADS) sample_top_p_kernel(const float* __restrict__ logits, int V,
                                                                       float temperature, float top_p,
                                                                       const float* __restrict__ u,
                                                                       int32_t* __restrict__ ids) {
  __shared__ SampleShared sh;
  pdl_wait();
  const int b = blockIdx.x;
  const float* row = logits + (size_t)b * V;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // max of z = logit / temperature
  float mx = -INFINITY;
  for (int i = threadIdx.x; i < V; i += blockDim.x) mx = fmaxf(mx, row[i] / temperature);
  mx = warp_max(mx);
  if (lane == 0) sh.red_f[warp] = mx;
  __syncthreads();
  if (warp == 0) {
    float t = lane < (int)(blockDim.x >> 5) ? sh.red_f[lane] : -INFINITY;
    t = warp_max(t);
    if (lane == 0) sh.red_f[0] = t;
  }
  __syncthreads();
  const float zmax = sh.red_f[0];
  // total integer mass W (exact)
  unsigned long long ws = 0;
  for (int i = threadIdx.x; i < V; i += blockDim.x) ws += token_mass(row[i] / temperature, zmax);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o);
  if (lane == 0) sh.red_u[warp] = ws;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += sh.red_u[w];
    sh.wsum = t;
  }
  __syncthreads();
  const unsigned long long W = sh.wsum;
  // the top-p cut: the token whose interval holds top_p * W is the last kept one
  unsigned long long kept = W;
  if (top_p < 1.0f) {
    const double tc = (double)top_p * (double)W;
    unsigned long long target = (unsigned long long)tc;
    if (target >= W) target = W - 1;
    select_by_mass(row, V, temperature, zmax, target, sh);
    kept = sh.sel_above + sh.sel_w;
    __syncthreads();
  }
  // the draw: the kept token whose interval holds u * kept
  float uu = u[b];
  uu = fminf(fmaxf(uu, 0.0f), 1.0f);
  unsigned long long target = (unsigned long long)((double)uu * (double)kept);
  if (target >= kept) target = kept - 1;
  select_by_mass(row, V, temperature, zmax, target, sh);
  if (threadIdx.x == 0) ids[b] = (int32_t)(0xFFFFFFFFu - (uint32_t)(sh.sel_prefix & 0xFFFFFFFFull));
}

}  // namespace llama
