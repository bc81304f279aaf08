// Bandwidth-bound kernels of the block: RMSNorm, fused RoPE + KV-cache
// append, embedding gather, last-row gather and greedy argmax.
#pragma once

#include "common.cuh"
#include "ragged.cuh"

namespace llama {

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// ------------------------------------------------------------------ RMSNorm (K1)
// h[m, :] = g * (x[m, :] * rsqrt(mean(x[m, :]^2) + eps)) ([MLX-13B] 4. RMSNorm;
// [DeepDive] LLaMARMSNorm).  One CTA per row; each thread keeps up to four
// 16-byte chunks of the row in registers, so the row is read from memory
// once; warp-shuffle then shared-memory reduction of the sum of squares.
// `x_row_stride` lets the final norm read the last row of each sequence
// only.  dim % 4 == 0, dim <= 16 * blockDim.x.
constexpr int RMS_MAX_V4 = 4;

inline int rmsnorm_threads(int dim) {
  int t = ((dim / 4 + RMS_MAX_V4 - 1) / RMS_MAX_V4 + 31) / 32 * 32;
  return t < 32 ? 32 : (t > 1024 ? 1024 : t);
}

// The RoPE angle of pair i at position pos, p * theta^(-2i/hd) ([DeepDive]
// LLaMARoPE), is formed and reduced modulo 2*pi in fp64; sincosf evaluates the
// reduced angle.  Shared by the stand-alone RoPE kernel and the per-token
// table the first RMSNorm writes for the fused QKV + RoPE GEMM epilogue.
__device__ __forceinline__ void rope_cos_sin(int pos, int i, int hd, float theta, float& c, float& s) {
  const double inv = pow((double)theta, -2.0 * (double)i / (double)hd);
  const double two_pi = 6.283185307179586476925286766559;
  double a = (double)pos * inv;
  a -= two_pi * floor(a / two_pi);
  sincosf((float)a, &s, &c);
}

// The rotation of one pair (x0, x1) by the angle with cosine c and sine s,
// rounded step by step (no contraction into fma), so that every kernel that
// applies RoPE to a decode token produces the same bits.
__device__ __forceinline__ float rope_lo(float x0, float x1, float c, float s) {
  return __fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, s));
}
__device__ __forceinline__ float rope_hi(float x0, float x1, float c, float s) {
  return __fadd_rn(__fmul_rn(x1, c), __fmul_rn(x0, s));
}

// Optional second output of an RMSNorm: per token row r (position p0 + r % L),
// tab[r * hd + i] = cos and tab[r * hd + hd/2 + i] = sin of pair i's angle.
struct RopeTab {
  float* tab;   // nullptr: none
  int hd, L, p0;
  float theta;
  int early_trigger;   // 1: signal dependents at entry (the next kernel is a GEMM)
};

template <typename OutT>
__global__ void __launch_bounds__(1024) rmsnorm_kernel(const float* __restrict__ x, long long x_row_stride,
                                                       const float* __restrict__ g, OutT* __restrict__ h, int rows,
                                                       int dim, float eps, RopeTab rt) {
  __shared__ float red[32];
  if (rt.early_trigger) pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  if (row >= rows) return;
  if (rt.tab != nullptr) {
    const int pos = rt.p0 + row % rt.L, hh = rt.hd >> 1;
    float* tr = rt.tab + (size_t)row * rt.hd;
    for (int i = threadIdx.x; i < hh; i += blockDim.x) rope_cos_sin(pos, i, rt.hd, rt.theta, tr[i], tr[hh + i]);
  }
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)row * x_row_stride);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  const int n4 = dim >> 2;
  float4 v[RMS_MAX_V4];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < RMS_MAX_V4; ++k) {
    const int i = threadIdx.x + k * blockDim.x;
    v[k] = i < n4 ? __ldg(xr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
  }
  ss = warp_sum(ss);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  if (warp == 0) {
    float t = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
    t = warp_sum(t);
    if (lane == 0) red[0] = t;
  }
  __syncthreads();
  const float rstd = rsqrtf(red[0] / (float)dim + eps);
  OutT* hr = h + (size_t)row * dim;
#pragma unroll
  for (int k = 0; k < RMS_MAX_V4; ++k) {
    const int i = threadIdx.x + k * blockDim.x;
    if (i >= n4) break;
    const float4 w = __ldg(g4 + i);
    const float a = w.x * (v[k].x * rstd), b = w.y * (v[k].y * rstd), c = w.z * (v[k].z * rstd),
                d = w.w * (v[k].w * rstd);
    if constexpr (sizeof(OutT) == 2) {
      uint2 o;
      o.x = pack_bf16x2(a, b);
      o.y = pack_bf16x2(c, d);
      reinterpret_cast<uint2*>(hr)[i] = o;
    } else {
      reinterpret_cast<float4*>(hr)[i] = make_float4(a, b, c, d);
    }
  }
}

// ------------------------------------------------------------------ RoPE + KV append (K3)
// One CTA per token.  The token's cos/sin ladder is computed once into shared
// memory: the angle p * theta^(-2i/hd) ([DeepDive] LLaMARoPE) is formed and
// reduced modulo 2*pi in fp64, then sincosf evaluates the reduced angle.
// Every (head, pair) of q and k is rotated; q is rotated in place in the
// projection buffer, rotated k and plain v are written to the cache at
// position p0 + t ([MLX-13B] KV 缓存实现片段: concatenate after the cached
// entries, RoPE offset = cache length).
//   qkv   [M, (nh + 2 nkv) hd] row-major (q | k | v), M = batch * L
//   cache [batch][nkv][cap][hd]
// style 0: rotate-half pairs (i, i + hd/2); style 1: adjacent pairs (2i, 2i+1).
// Each thread moves 16 bytes at a time (8 bf16 or 4 fp32 elements).
// A ragged batch (tab != nullptr): token m is row m - start[b] of sequence b
// = seq_of_row(m), at position p0[b] + that row.
template <typename T>
__global__ void __launch_bounds__(256) rope_append_kernel(T* __restrict__ qkv, T* __restrict__ kc,
                                                          T* __restrict__ vc, int L, int p0, int nh, int nkv,
                                                          int hd, int cap, float theta, int style,
                                                          const SeqTab* __restrict__ tab) {
  constexpr int VE = 16 / sizeof(T);      // elements per 16-byte vector
  __shared__ float cs[64], sn[64];
  const int m = blockIdx.x;
  int b, p;
  if (tab == nullptr) {
    b = m / L;
    p = p0 + m % L;
  } else {
    pdl_wait();   // the table is written by the kernel before
    b = seq_of_row(tab, m);
    p = tab->p0[b] + (m - tab->start[b]);
  }
  const int half = hd >> 1;
  for (int i = threadIdx.x; i < half; i += blockDim.x) rope_cos_sin(p, i, hd, theta, cs[i], sn[i]);
  __syncthreads();
  pdl_wait();
  const int qkvn = (nh + 2 * nkv) * hd;
  T* row = qkv + (size_t)m * qkvn;
  const int heads = nh + nkv;
  if (style == 0) {
    // rotate-half: a vector of VE elements at i (first half) pairs with the one at i + half
    const int vph = half / VE;                        // vectors per half head
    for (int e = threadIdx.x; e < heads * vph; e += blockDim.x) {
      const int head = e / vph, i0 = (e % vph) * VE;
      T* hv = row + head * hd;
      uint4 ua = *reinterpret_cast<const uint4*>(hv + i0);
      uint4 ub = *reinterpret_cast<const uint4*>(hv + i0 + half);
      T* xa = reinterpret_cast<T*>(&ua);
      T* xb = reinterpret_cast<T*>(&ub);
#pragma unroll
      for (int k = 0; k < VE; ++k) {
        const float x0 = to_f32(xa[k]), x1 = to_f32(xb[k]);
        const float c = cs[i0 + k], s = sn[i0 + k];
        xa[k] = from_f32<T>(rope_lo(x0, x1, c, s));
        xb[k] = from_f32<T>(rope_hi(x0, x1, c, s));
      }
      T* dst = hv;
      if (head >= nh) dst = kc + (((size_t)b * nkv + (head - nh)) * cap + p) * hd;
      *reinterpret_cast<uint4*>(dst + i0) = ua;
      *reinterpret_cast<uint4*>(dst + i0 + half) = ub;
    }
  } else {
    // interleaved: a vector holds VE/2 adjacent pairs
    const int vpr = hd / VE;                          // vectors per head row
    for (int e = threadIdx.x; e < heads * vpr; e += blockDim.x) {
      const int head = e / vpr, i0 = (e % vpr) * VE;
      T* hv = row + head * hd;
      uint4 u = *reinterpret_cast<const uint4*>(hv + i0);
      T* x = reinterpret_cast<T*>(&u);
#pragma unroll
      for (int k = 0; k < VE; k += 2) {
        const float x0 = to_f32(x[k]), x1 = to_f32(x[k + 1]);
        const int pi = (i0 + k) >> 1;
        const float c = cs[pi], s = sn[pi];
        x[k] = from_f32<T>(rope_lo(x0, x1, c, s));
        x[k + 1] = from_f32<T>(rope_hi(x0, x1, c, s));
      }
      T* dst = hv;
      if (head >= nh) dst = kc + (((size_t)b * nkv + (head - nh)) * cap + p) * hd;
      *reinterpret_cast<uint4*>(dst + i0) = u;
    }
  }
  // copy v
  const int vpr = hd / VE;
  const T* vsrc = row + (nh + nkv) * hd;
  for (int e = threadIdx.x; e < nkv * vpr; e += blockDim.x) {
    const int gkv = e / vpr, i0 = (e % vpr) * VE;
    *reinterpret_cast<uint4*>(vc + (((size_t)b * nkv + gkv) * cap + p) * hd + i0) =
        *reinterpret_cast<const uint4*>(vsrc + gkv * hd + i0);
  }
}

// ------------------------------------------------------------------ embedding gather (K6)
// x[m, :] = float(E[tok[m], :]) ([DeepDive] class LLaMA: nn.Embedding).
// One warp per token, 16-byte loads.  Out-of-range ids record INVALID_ARG
// in the status word and produce a zero row.
template <typename T>
__global__ void __launch_bounds__(256) embed_kernel(const int32_t* __restrict__ tok, const T* __restrict__ E,
                                                    float* __restrict__ x, int M, int dim, int vocab,
                                                    DevStatus* st) {
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= M) return;
  const int id = tok[warp];
  float* xr = x + (size_t)warp * dim;
  if (id < 0 || id >= vocab) {
    if (lane == 0) record_error(st, LLAMA_ERR_INVALID_ARG, 20, warp);
    for (int i = lane; i < dim; i += 32) xr[i] = 0.f;
    return;
  }
  const T* er = E + (size_t)id * dim;
  if constexpr (sizeof(T) == 2) {
    for (int i = lane; i < dim / 8; i += 32) {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(er) + i);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
      float4 a, b;
      float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
      float2 f2 = __bfloat1622float2(h2[2]), f3 = __bfloat1622float2(h2[3]);
      a = make_float4(f0.x, f0.y, f1.x, f1.y);
      b = make_float4(f2.x, f2.y, f3.x, f3.y);
      reinterpret_cast<float4*>(xr)[2 * i] = a;
      reinterpret_cast<float4*>(xr)[2 * i + 1] = b;
    }
  } else {
    for (int i = lane; i < dim / 4; i += 32)
      reinterpret_cast<float4*>(xr)[i] = __ldg(reinterpret_cast<const float4*>(er) + i);
  }
}

// ------------------------------------------------------------------ greedy argmax (K7)
// ids[b] = argmax_v logits[b, v]; ties resolve to the lowest index
// ([HandsOn] 第三章: argmax of the last position; numpy/torch convention).
// One CTA per row; NaN never wins.
__global__ void __launch_bounds__(1024) argmax_kernel(const float* __restrict__ logits, int vocab,
                                                      int32_t* __restrict__ ids) {
  pdl_wait();
  const int b = blockIdx.x;
  const float* r = logits + (size_t)b * vocab;
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int v = threadIdx.x; v < vocab; v += blockDim.x) {
    const float x = r[v];
    if (x > best || (x == best && v < bi)) {
      best = x;
      bi = v;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ob > best || (ob == best && oi < bi)) {
      best = ob;
      bi = oi;
    }
  }
  __shared__ float sb[32];
  __shared__ int si[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sb[warp] = best;
    si[warp] = bi;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    best = lane < nw ? sb[lane] : -INFINITY;
    bi = lane < nw ? si[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) {
        best = ob;
        bi = oi;
      }
    }
    if (lane == 0) ids[b] = bi == 0x7fffffff ? 0 : bi;
  }
}

// Gather the last row of each of `batch` sequences of length L: dst[b] = src[b*L + L-1].
__global__ void gather_last_rows_kernel(const float* __restrict__ src, float* __restrict__ dst, int L, int dim) {
  pdl_wait();
  const int b = blockIdx.y;
  const float* s = src + ((size_t)b * L + (L - 1)) * dim;
  float* d = dst + (size_t)b * dim;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < dim; i += gridDim.x * blockDim.x) d[i] = s[i];
}

// Copy a ragged batch's table (kernel parameter) into the workspace, where the
// call's later kernels read it.
__global__ void seqtab_kernel(const __grid_constant__ SeqTab t, SeqTab* __restrict__ dst) {
  pdl_wait();   // earlier kernels may still read the previous call's table
  if (threadIdx.x == 0) dst->n = t.n;
  for (int i = threadIdx.x; i < t.n; i += blockDim.x) {
    dst->start[i] = t.start[i];
    dst->len[i] = t.len[i];
    dst->p0[i] = t.p0[i];
  }
}

// Device-side failure self-test: wait on an mbarrier that nothing arrives on;
// the bounded wait runs out, records LLAMA_ERR_DEVICE_TIMEOUT and returns.
__global__ void selftest_wait_kernel(DevStatus* st, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtx wc{&abort_sh, st, limit_ns, 99};
    mbar_wait(smem_u32(&bar), 0, wc, 0);
  }
}

}  // namespace llama
