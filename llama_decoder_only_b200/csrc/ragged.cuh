// Per-call table of a ragged batch (sequences with their own cache lengths
// and numbers of new tokens).
#pragma once

#include "common.cuh"

namespace llama {

// Per-call table of a ragged batch ([MLX-13B] KV 缓存实现片段 keeps one offset,
// key_cache.shape[2], for the whole batch; here every sequence keeps its own):
// sequence b brings len[b] new tokens, packed at rows start[b] .. start[b] +
// len[b] - 1 of the call's activations, at positions p0[b] .. p0[b] + len[b] - 1
// (p0[b] = its cache length before the call).  Kernels read it from the
// workspace (written by seqtab_kernel at the start of the call); a null
// pointer means the uniform batch of the kernel's own parameters.
constexpr int kMaxRagged = 128;

struct SeqTab {
  int n;
  int start[kMaxRagged];
  int len[kMaxRagged];
  int p0[kMaxRagged];
};

// Sequence of packed row m (start[] ascending, start[0] = 0).
__device__ __forceinline__ int seq_of_row(const SeqTab* t, int m) {
  int lo = 0, hi = t->n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (t->start[mid] <= m) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace llama
