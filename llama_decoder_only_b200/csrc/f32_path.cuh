// fp32 path of the block (dtype LLAMA_F32): CUDA-core GEMMs with fused
// epilogues and a CUDA-core causal GQA attention.  fp32 FMA only (no TF32),
// so the result stays within a few fp32 ulps of the exact definition.
#pragma once

#include "common.cuh"

namespace llama {

enum F32Epi : int { F32_STORE = 0, F32_RESID = 1, F32_SWIGLU = 2 };

// out[m, n] = epi(sum_k A[m, k] * B[n, k]); 64x64 output tile per CTA,
// 256 threads x (4 x 4) outputs, K staged through shared memory 16 at a time.
// F32_SWIGLU keeps two accumulators (B0 = gate rows, B1 = up rows) and stores
// silu(gate) * up ([MLX-13B] 3. 前馈网络; [DeepDive] LLaMAMLP).
template <int EPI>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, int lda,
                                                       const float* __restrict__ B0,
                                                       const float* __restrict__ B1, int ldb, int M, int N,
                                                       int K, float* __restrict__ out, int ldo,
                                                       const float* __restrict__ resid, int ldr) {
  constexpr int TM = 64, TN = 64, TK = 16;
  constexpr int NB = EPI == F32_SWIGLU ? 2 : 1;
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[NB][TK][TN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  float acc[NB][4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int e = threadIdx.x; e < TM * TK; e += 256) {
      const int r = e / TK, c = e % TK;
      const int m = m0 + r, k = k0 + c;
      As[c][r] = (m < M && k < K) ? A[(size_t)m * lda + k] : 0.f;
    }
    for (int e = threadIdx.x; e < TN * TK; e += 256) {
      const int r = e / TK, c = e % TK;
      const int n = n0 + r, k = k0 + c;
      Bs[0][c][r] = (n < N && k < K) ? B0[(size_t)n * ldb + k] : 0.f;
      if (NB == 2) Bs[NB - 1][c][r] = (n < N && k < K) ? B1[(size_t)n * ldb + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int s = 0; s < NB; ++s)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float bv = Bs[s][kk][tx * 4 + j];
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[s][i][j] = fmaf(a[i], bv, acc[s][i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v;
      if (EPI == F32_SWIGLU) {
        v = silu_f(acc[0][i][j]) * acc[NB - 1][i][j];
      } else {
        v = acc[0][i][j];
        if (EPI == F32_RESID) v += resid[(size_t)m * ldr + n];
      }
      out[(size_t)m * ldo + n] = v;
    }
  }
}

// Causal GQA attention, fp32, one CTA (128 threads) per (query row, head,
// sequence).  Scores for the visible keys j <= p go to shared memory, then
// max, exp-sum and the weighted sum of V ([MLX-13B] 2. 注意力机制,
// 5. 因果掩码; [DeepDive] LLaMAAttention with kv head = h / n_rep).
//   q   [M, ld_q] with head h at columns h*hd (rows b*L + t)
//   kc, vc [batch][nkv][cap][hd]; out [M, nh*hd]
__global__ void __launch_bounds__(128) attn_f32_kernel(const float* __restrict__ q, int ld_q,
                                                       const float* __restrict__ kc, const float* __restrict__ vc,
                                                       float* __restrict__ out, int L, int p0, int nh, int nkv,
                                                       int hd, int cap) {
  extern __shared__ float sc[];  // [p + 1] scores, then reduction scratch
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int m = b * L + t;
  const int p = p0 + t;
  const int T = p + 1;
  const int g = h / (nh / nkv);
  const float* qr = q + (size_t)m * ld_q + h * hd;
  const float* K = kc + ((size_t)b * nkv + g) * cap * hd;
  const float* V = vc + ((size_t)b * nkv + g) * cap * hd;
  const float scale = rsqrtf((float)hd);
  __shared__ float red[32];
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < T; j += blockDim.x) {
    const float* kr = K + (size_t)j * hd;
    float s = 0.f;
    for (int d = 0; d < hd; ++d) s = fmaf(qr[d], kr[d], s);
    s *= scale;
    sc[j] = s;
    mx = fmaxf(mx, s);
  }
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j < T; j += blockDim.x) {
    const float e = expf(sc[j] - mx);
    sc[j] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  sum = red[0] + red[1] + red[2] + red[3];
  const float inv = 1.0f / sum;
  for (int d = threadIdx.x; d < hd; d += blockDim.x) {
    float o = 0.f;
    for (int j = 0; j < T; ++j) o = fmaf(sc[j], V[(size_t)j * hd + d], o);
    out[(size_t)m * nh * hd + h * hd + d] = o * inv;
  }
}

}  // namespace llama
