// C-ABI host library: argument checks, workspace layout, tensor maps and the
// launch sequence of one decoder block (prefill / decode) and of a whole
// model.  Every step of the block runs in the kernels of this library; the
// host only validates, plans and enqueues.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <set>
#include <tuple>
#include <utility>
#include <unordered_map>
#include <vector>

#include "attention.cuh"
#include "common.cuh"
#include "decode_layer.cuh"
#include "f32_path.cuh"
#include "gemm_q4.cuh"
#include "gemm_tc.cuh"
#include "sampling.cuh"
#include "small_kernels.cuh"

using namespace llama;

struct llama_kv_cache {
  llama_dims dims;
  int32_t batch;
  int32_t capacity;
  int32_t length;              // common length of every sequence; -2 while the lengths differ
  std::vector<int32_t> lens;   // per-sequence lengths while they differ (empty: all are `length`)
  void* k;
  void* v;
};

namespace {

std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
constexpr int kMaxSkGrid = 192;     // upper bound on stream-K CTAs (workspace sizing)
constexpr int kMaxAttnSplits = 64;  // upper bound on decode attention splits
// workspace header (see plan_ws): status word, the decode GEMMs' flags and the
// fused RMSNorm's counters (the rest of the 4 KB is reserved)
constexpr size_t kWsFlagsOffset = 256;
constexpr size_t kWsNormCtrOffset = 1024;   // [2]: the fused RMSNorm's tile and CTA counters
constexpr size_t kWsGridBarOffset = 1056;   // [8]: the persistent decode block's grid barriers
constexpr size_t kWsHeaderBytes = 4096;
static_assert(kWsFlagsOffset + kMaxSkGrid * 4 <= kWsNormCtrOffset, "GEMM flags overflow their area");
constexpr int kMaxNormTiles = 512;           // tiles of a residual GEMM with a fused RMSNorm
constexpr int kSwapMaxTokens = 128; // decode GEMMs use the swapped stream-K form up to here

// ------------------------------------------------------------------ tracing
// Every kernel launch of the library is counted; when tracing is on it is
// also bracketed by two CUDA events on its stream, and llama_profile_read
// sums the elapsed times per kernel kind.

enum KernelKind : int {
  K_RMSNORM = 0, K_GEMM_QKV, K_ROPE_APPEND, K_ATTN_PREFILL, K_ATTN_DECODE, K_ATTN_COMBINE, K_GEMM_O,
  K_GEMM_GATE_UP, K_GEMM_DOWN, K_EMBED, K_GATHER_LAST, K_GEMM_LM_HEAD, K_ARGMAX,
  K_GEMM_F32, K_ATTN_F32, K_SELFTEST, K_SAMPLE, K_SEQTAB, K_DECODE_LAYER, K_COUNT
};
const char* const kKindNames[K_COUNT] = {
  "rmsnorm", "gemm_qkv", "rope_kv_append", "attn_prefill", "attn_decode", "attn_decode_combine", "gemm_o_proj",
  "gemm_gate_up_swiglu", "gemm_down", "embed", "gather_last_rows", "gemm_lm_head", "argmax",
  "gemm_f32", "attn_f32", "selftest", "sample_top_p", "seq_table", "decode_layer"};

struct ProfRec {
  cudaEvent_t a, b;
  int kind;
};

struct Tracer {
  std::mutex mu;
  bool on = false;
  std::vector<ProfRec> pending;
  double total_ms[K_COUNT] = {};
  long long launches[K_COUNT] = {};
};
Tracer& tracer() {
  static Tracer t;
  return t;
}
std::atomic<unsigned long long> g_launch_count{0};

// LLAMA_SYNC_TRACE=1 (debugging aid): print every launch to stderr and wait
// for it to finish before returning, so a failing kernel is named.
bool sync_trace() {
  static const bool on = [] {
    const char* e = std::getenv("LLAMA_SYNC_TRACE");
    return e != nullptr && e[0] == '1';
  }();
  return on;
}

struct LaunchScope {
  cudaStream_t st;
  int kind;
  cudaEvent_t a = nullptr, b = nullptr;
  LaunchScope(cudaStream_t s, int k) : st(s), kind(k) {
    g_launch_count.fetch_add(1, std::memory_order_relaxed);
    if (sync_trace()) std::fprintf(stderr, "[llama] launch %s\n", kKindNames[kind]);
    Tracer& t = tracer();
    if (t.on && cudaEventCreate(&a) == cudaSuccess && cudaEventCreate(&b) == cudaSuccess) {
      cudaEventRecord(a, st);
    } else {
      a = b = nullptr;
    }
  }
  ~LaunchScope() {
    if (sync_trace()) {
      const cudaError_t e = cudaStreamSynchronize(st);
      std::fprintf(stderr, "[llama] done %s: %s\n", kKindNames[kind], cudaGetErrorString(e));
    }
    if (a != nullptr) {
      cudaEventRecord(b, st);
      Tracer& t = tracer();
      std::lock_guard<std::mutex> g(t.mu);
      t.pending.push_back({a, b, kind});
    }
  }
};
#define TRACE(kind, stream) LaunchScope _trace_scope_(stream, kind)

// (with LLAMA_SYNC_TRACE=1 the failing call and its error are printed)
#define CUDA_TRY(x)                                                                  \
  do {                                                                               \
    const cudaError_t cuda_try_e = (x);                                              \
    if (cuda_try_e != cudaSuccess) {                                                 \
      if (sync_trace()) std::fprintf(stderr, "[llama] %s: %s\n", #x, cudaGetErrorString(cuda_try_e)); \
      (void)cudaGetLastError();                                                      \
      return LLAMA_ERR_CUDA;                                                         \
    }                                                                                \
  } while (0)

#define LAUNCH_CHECK()                                                               \
  do {                                                                               \
    const cudaError_t launch_check_e = cudaGetLastError();                           \
    if (launch_check_e != cudaSuccess) {                                             \
      if (sync_trace()) std::fprintf(stderr, "[llama] launch: %s\n", cudaGetErrorString(launch_check_e)); \
      return LLAMA_ERR_CUDA;                                                         \
    }                                                                                \
  } while (0)

#define TRY(x)                                \
  do {                                        \
    llama_status _s = (x);                    \
    if (_s != LLAMA_OK) return _s;            \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

// ------------------------------------------------------------------ driver entry point for tensor maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 tensor map, 128-byte swizzle, zero fill out of bounds.
// dims[0] is the contiguous dimension; strides are in bytes for dims 1..rank-1.
bool make_map_ex(CUtensorMap* m, const void* base, CUtensorMapDataType dt, CUtensorMapSwizzle sw, int rank,
                 const uint64_t* dims, const uint64_t* strides, const uint32_t* box) {
  auto enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t d[5], s[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides[i];
  CUresult r = enc(m, dt, (cuuint32_t)rank, const_cast<void*>(base), d, s, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box) {
  return make_map_ex(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_128B, rank, dims, strides, box);
}

// Encoded 2-D maps are cached by (base, inner, rows, box rows): weights and
// workspace buffers recur every call, and encoding is host work on the
// launch path.  The cache is cleared when it grows past a bound.
struct MapKey {
  uintptr_t base;
  uint64_t inner, rows;
  uint32_t box_rows;
  bool operator==(const MapKey& o) const {
    return base == o.base && inner == o.inner && rows == o.rows && box_rows == o.box_rows;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    uint64_t h = k.base * 0x9E3779B97F4A7C15ull;
    h ^= (k.inner + 0x632BE59BD9B4E019ull) * 0xC2B2AE3D27D4EB4Full + (h << 6) + (h >> 2);
    h ^= (k.rows * 31 + k.box_rows) * 0x165667B19E3779F9ull + (h << 6) + (h >> 2);
    return (size_t)h;
  }
};

bool make_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  static std::mutex mu;
  static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
  const MapKey key{reinterpret_cast<uintptr_t>(base), inner, rows, box_rows};
  {
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *m = it->second;
      return true;
    }
  }
  const uint64_t dims[2] = {inner, rows};
  const uint64_t strides[1] = {inner * 2};
  const uint32_t box[2] = {64, box_rows};
  if (!make_map(m, base, 2, dims, strides, box)) return false;
  std::lock_guard<std::mutex> g(mu);
  if (cache.size() > 8192) cache.clear();
  cache.emplace(key, *m);
  return true;
}

int num_sms() {
  static int cached[64] = {};
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return 148;
  }
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

// Launch with programmatic stream serialization (the kernels call pdl_trigger /
// pdl_wait), so a kernel's prologue overlaps the tail of the one before it.
// LLAMA_NO_PDL=1 launches them in plain stream order instead.
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("LLAMA_NO_PDL");
    return !(e != nullptr && e[0] == '1');
  }();
  return on;
}

// LLAMA_DECODE_SPLITS=n (n >= 1): use n key splits in the decode attention
// instead of the heuristic's count (clamped to the kernel's limits).
int forced_decode_splits() {
  static const int n = [] {
    const char* e = std::getenv("LLAMA_DECODE_SPLITS");
    return e != nullptr ? std::atoi(e) : 0;
  }();
  return n;
}

// Which decode-attention kernel serves (head_dim, GQA group): the TMA-fed
// tensor-core kernel for groups >= 4 (its 16-row tile fills) and for head_dim
// 96 (where the CUDA-core kernel's 24 elements a lane hold two CTAs per SM:
// Phi-3-mini-shaped block, batch 8, cache 512: 16.8 vs 21.5 us), the CUDA-core
// one otherwise.  LLAMA_DECODE_ATTN=mma | simt forces one of them.
// LLAMA_DECODE_ATTN: 1 = mma, 2 = simt, 0 = not set.
int decode_attn_forced() {
  static const int forced = [] {
    const char* e = std::getenv("LLAMA_DECODE_ATTN");
    if (e == nullptr) return 0;
    return std::strcmp(e, "mma") == 0 ? 1 : (std::strcmp(e, "simt") == 0 ? 2 : 0);
  }();
  return forced;
}

bool use_decode_mma(int hd, int grp) {
  if (decode_attn_forced() == 1) return true;
  if (decode_attn_forced() == 2) return false;
  return (grp >= 4 && (hd == 64 || hd == 128)) || hd == 96;
}

// LLAMA_EARLY_TRIGGER=1: the decode GEMMs, RMSNorm and the split combine signal
// their dependents at entry instead of at the end of their work.
int early_trigger() {
  static const int on = [] {
    const char* e = std::getenv("LLAMA_EARLY_TRIGGER");
    return (e != nullptr && e[0] == '1') ? 1 : 0;
  }();
  return on;
}


template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same for a kernel whose CTAs run in 2-CTA clusters (tcgen05 CTA pairs); grid.x is even.
template <typename... KArgs, typename... Args>
cudaError_t launch_k_pair(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same for a kernel whose CTAs run in clusters of `cl` CTAs along x; grid.x is a multiple of cl.
template <typename... KArgs, typename... Args>
cudaError_t launch_k_cluster(void (*kernel)(KArgs...), int cl, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// cudaFuncSetAttribute acts on the current device only, so a kernel's dynamic
// shared-memory limit is raised once per (kernel, device) pair.
llama_status ensure_smem_attr(const void* kernel, int bytes) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  std::lock_guard<std::mutex> g(mu);
  if (done.count({kernel, dev}) != 0) return LLAMA_OK;
  CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  done.insert({kernel, dev});
  return LLAMA_OK;
}

// ------------------------------------------------------------------ validation

llama_status check_dims(const llama_dims* d) {
  if (d == nullptr) return LLAMA_ERR_INVALID_ARG;
  if (d->dim <= 0 || d->n_heads <= 0 || d->n_kv_heads <= 0 || d->head_dim <= 0 || d->ffn_dim <= 0)
    return LLAMA_ERR_INVALID_ARG;
  if (d->n_heads % d->n_kv_heads != 0) return LLAMA_ERR_INVALID_ARG;
  if (!(d->eps > 0.f) || !(d->eps < 1.f)) return LLAMA_ERR_INVALID_ARG;
  if (!(d->rope_theta > 1.f) || !(d->rope_theta < 1e30f)) return LLAMA_ERR_INVALID_ARG;
  if (d->rope_style != LLAMA_ROPE_HALF && d->rope_style != LLAMA_ROPE_INTERLEAVED) return LLAMA_ERR_INVALID_ARG;
  if (d->dtype != LLAMA_F32 && d->dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARG;
  if (d->dim % 8 || d->ffn_dim % 8) return LLAMA_ERR_UNSUPPORTED;
  if (d->dim > 16 * 1024) return LLAMA_ERR_UNSUPPORTED;   // RMSNorm keeps a row in one CTA's registers
  const int hd = d->head_dim;
  if (d->dtype == LLAMA_BF16) {
    if (hd != 64 && hd != 96 && hd != 128) return LLAMA_ERR_UNSUPPORTED;
    const int grp = d->n_heads / d->n_kv_heads;
    if (grp != 1 && grp != 2 && grp != 4 && grp != 8) return LLAMA_ERR_UNSUPPORTED;
  } else {
    if (hd != 32 && hd != 64 && hd != 96 && hd != 128) return LLAMA_ERR_UNSUPPORTED;
  }
  return LLAMA_OK;
}

bool same_dims(const llama_dims& a, const llama_dims& b) { return std::memcmp(&a, &b, sizeof(llama_dims)) == 0; }

llama_status check_weights(const llama_layer_weights* w) {
  if (w == nullptr) return LLAMA_ERR_INVALID_ARG;
  const void* ps[9] = {w->attn_norm, w->wq, w->wk, w->wv, w->wo, w->ffn_norm, w->w1, w->w3, w->w2};
  for (const void* p : ps)
    if (p == nullptr) return LLAMA_ERR_INVALID_ARG;
  for (const void* p : ps)
    if (!aligned16(p)) return LLAMA_ERR_ALIGNMENT;
  return LLAMA_OK;
}

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// ------------------------------------------------------------------ workspace layout

struct WsLayout {
  size_t qkv, h, attn, mbuf, partial, sk_flags, att_ml, att_o, rope_tab, seqtab, ssq;   // layer scratch
  size_t xa, xb, xl, hl, logits;                            // model scratch
  size_t total;
};

int swap_bn(int tokens) { return tokens <= 16 ? 16 : tokens <= 32 ? 32 : tokens <= 64 ? 64 : 128; }

// Stream-K partial buffer of one decode GEMM (floats): one [128][BN] piece per CTA.
size_t sk_partial_floats(int tokens) { return (size_t)kMaxSkGrid * swap_bn(tokens) * 128; }

// ragged_tokens >= 0: a ragged batch of `batch` sequences with that many new
// tokens in all (seq_len unused); it adds the sequence table at the end.
WsLayout plan_ws(const llama_dims& d, int batch, int seq_len, int vocab, int ragged_tokens = -1) {
  WsLayout w{};
  const size_t es = d.dtype == LLAMA_BF16 ? 2 : 4;
  const bool ragged = ragged_tokens >= 0;
  const size_t M = ragged ? (size_t)ragged_tokens : (size_t)batch * seq_len;
  const int sk_tokens = ragged ? ragged_tokens : batch;   // token rows of the swapped decode GEMMs
  const int qkvn = (d.n_heads + 2 * d.n_kv_heads) * d.head_dim;
  // Fixed header, the same for every (batch, seq_len): the words that must
  // read zero when a launch starts -- the status word and the decode GEMMs'
  // per-CTA flags.  Every launch leaves them zero; the tensors after the
  // header move with the call's shape, so one call's data never lands on
  // another call's flags.
  w.sk_flags = kWsFlagsOffset;
  size_t off = kWsHeaderBytes;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  w.qkv = take(M * qkvn * es);
  w.h = take(M * (size_t)d.dim * es);
  w.attn = take(M * (size_t)d.n_heads * d.head_dim * es);
  w.mbuf = take(M * (size_t)d.ffn_dim * es);
  // decode GEMMs (M = batch) and the lm_head on the last rows (M = batch)
  const bool sk = d.dtype == LLAMA_BF16 && sk_tokens <= kSwapMaxTokens;
  w.partial = take(sk ? sk_partial_floats(sk_tokens) * 4 : 0);

  w.att_ml = take((size_t)batch * d.n_heads * kMaxAttnSplits * 2 * 4);
  w.att_o = take((size_t)batch * d.n_heads * kMaxAttnSplits * d.head_dim * 4);
  // per-token cos/sin for the prefill QKV GEMM with RoPE fused in
  const bool rope_fused = d.dtype == LLAMA_BF16 && (d.head_dim == 64 || d.head_dim == 128);
  w.rope_tab = take(rope_fused ? M * (size_t)d.head_dim * 4 : 0);
  if (vocab > 0) {
    w.xa = take(M * (size_t)d.dim * 4);
    w.xb = take(M * (size_t)d.dim * 4);
    w.xl = take((size_t)batch * d.dim * 4);
    w.hl = take((size_t)batch * d.dim * es);
    w.logits = take((size_t)batch * vocab * 4);
  }
  w.seqtab = take(ragged ? sizeof(SeqTab) : 0);
  // per-tile sums of squares of the decode residual GEMMs with the next RMSNorm fused in
  // (+ [CTA][16] shares of the persistent decode block's first RMSNorm)
  w.ssq = take(sk ? ((size_t)kMaxNormTiles * swap_bn(sk_tokens) + (size_t)kMaxSkGrid * 16) * 4 : 0);
  w.total = off;
  return w;
}

// ------------------------------------------------------------------ GEMM launchers (bf16, tcgen05)

struct WSeg {
  const void* ptr;
  int rows;
  int col0;
};

template <int BN, bool SWAP, int EPI, int KS = 1>
llama_status launch_gemm_tc(const CUtensorMap& a, const CUtensorMap* w, const GemmParams& p, int grid,
                            cudaStream_t st, int kind) {
  using C = GemmCfg<BN, !SWAP, KS>;
  TRY(ensure_smem_attr(reinterpret_cast<const void*>(gemm_tc_kernel<BN, SWAP, EPI, KS>), C::SMEM_BYTES));
  {
    TRACE(kind, st);
    if (SWAP)
      CUDA_TRY(launch_k(gemm_tc_kernel<BN, SWAP, EPI, KS>, grid, GEMM_THREADS, C::SMEM_BYTES, st, a, w[0], w[1], w[2],
                        p));
    else
      CUDA_TRY(launch_k_pair(gemm_tc_kernel<BN, SWAP, EPI, KS>, grid, GEMM_THREADS, C::SMEM_BYTES, st, a, w[0], w[1],
                             w[2], p));
  }
  LAUNCH_CHECK();
  return LLAMA_OK;
}

// k sub-blocks of 64 per decode GEMM unit (LLAMA_DECODE_KSUB=1 or 2, default 2):
// 2 makes every stage read 256 contiguous bytes of each weight row.
int decode_ksub() {
  static const int ks = [] {
    const char* e = std::getenv("LLAMA_DECODE_KSUB");
    return (e != nullptr && e[0] == '1') ? 1 : 2;
  }();
  return ks;
}

// Stream-K scratch of the decode GEMMs: one fp32 piece and one flag per CTA.
struct SkScratch {
  float* partial;
  unsigned* flags;   // the workspace header's flag area (chunk and tile counters follow it)
  float* ssq;        // per-tile sums of squares for a fused RMSNorm
};

// An RMSNorm fused into the end of a decode residual GEMM: out = bf16(g * x * rstd(x row)).
struct NormFuse {
  const float* g;
  void* out;
  float eps;
};

// An RMSNorm computed by the decode GEMM that consumes it (cluster form): its
// B operand is bf16(g * x * rstd(x row)), rstd from the sums of squares that
// the residual GEMM which wrote x left in `ssq` ([tiles][BN]).
struct NormB {
  const float* x;
  int ldx;
  const float* g;
  const float* ssq;
  int tiles;
  int dim;
  float eps;
  void* h;   // bf16 [rows][dim]: the normalised rows are also stored here (nullptr: not)
};

// Cluster-split form of a decode GEMM: one weight tile per cluster of p.cl_split CTAs.
template <int BN, int EPI>
llama_status launch_gemm_cl(const CUtensorMap& a, const CUtensorMap* w, const GemmParams& p, int grid,
                            cudaStream_t st, int kind) {
  using C = GemmCfg<BN, false, 2, true>;
  auto* k = gemm_tc_kernel<BN, true, EPI, 2, true>;
  TRY(ensure_smem_attr(reinterpret_cast<const void*>(k), C::SMEM_BYTES));
  {
    TRACE(kind, st);
    CUDA_TRY(launch_k_cluster(k, p.cl_split, grid, GEMM_THREADS, C::SMEM_BYTES, st, a, w[0], w[1], w[2], p));
  }
  LAUNCH_CHECK();
  return LLAMA_OK;
}

// Largest cluster the CL kernel of this width can reduce in shared memory
// (the form exists for up to 16 token rows).
int cl_max_split(int BN) { return BN == 16 ? kMaxClusterSplit : 0; }

// True when every cluster of `cl` CTAs of the CL kernel (BN, epi) fits on the
// device at once (`clusters` of them).  Cached per (BN, epi, cl, device).
bool clusters_fit(int BN, int epi, int cl, int clusters) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int>, int> cache;
  std::lock_guard<std::mutex> g(mu);
  const auto key = std::make_tuple(BN, epi, cl, dev);
  auto it = cache.find(key);
  if (it == cache.end()) {
    const void* k = nullptr;
    int smem = 0;
    auto pick = [&](auto kern, int bytes) {
      k = reinterpret_cast<const void*>(kern);
      smem = bytes;
    };
    using C = GemmCfg<16, false, 2, true>;
    if (epi == EPI_BF16) pick(gemm_tc_kernel<16, true, EPI_BF16, 2, true>, C::SMEM_BYTES);
    else if (epi == EPI_RESID_F32) pick(gemm_tc_kernel<16, true, EPI_RESID_F32, 2, true>, C::SMEM_BYTES);
    else pick(gemm_tc_kernel<16, true, EPI_SWIGLU_BF16, 2, true>, C::SMEM_BYTES);
    int n = 0;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3((unsigned)(cl * clusters));
      cfg.blockDim = dim3(GEMM_THREADS);
      cfg.dynamicSmemBytes = (size_t)smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)cl;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    it = cache.emplace(key, n).first;
  }
  return it->second >= clusters;
}

// A decode GEMM of at most 16 token rows whose weight tiles number at most
// the SM count runs as one cluster per tile, its k-blocks split over the
// cluster's CTAs and their pieces added in the rank-0 CTA's shared memory
// instead of through L2 and flags, when that keeps at least 3/4 of the SMs
// busy.  LLAMA_DECODE_CLUSTER=0 keeps every decode GEMM stream-K; =2 takes
// clusters whatever the SM share (tests of small shapes).  Returns the
// cluster size, 0 for stream-K.
int decode_cluster_split(int n_tiles, int num_kb, int BN, int KS, int epi) {
  static const int mode = [] {
    const char* e = std::getenv("LLAMA_DECODE_CLUSTER");
    return e == nullptr ? 1 : e[0] == '0' ? 0 : e[0] == '2' ? 2 : 1;
  }();
  // LLAMA_DECODE_CLUSTER_MIN=s: use clusters of at least s CTAs only
  static const int min_split = [] {
    const char* e = std::getenv("LLAMA_DECODE_CLUSTER_MIN");
    const int v = e != nullptr ? std::atoi(e) : 1;
    return v < 1 ? 1 : v;
  }();
  if (mode == 0 || KS != 2 || epi == EPI_F32 || cl_max_split(BN) < 1 || n_tiles <= 0) return 0;
  const int sms = num_sms();
  auto busy = [&](int S) { return mode == 2 || 4 * n_tiles * S >= 3 * sms; };
  int S = std::min({cl_max_split(BN), sms / n_tiles, num_kb});
  if (S < min_split || !busy(S)) return 0;
  while (S >= min_split && !clusters_fit(BN, epi, S, n_tiles)) --S;
  if (S < min_split || !busy(S)) return 0;
  return S;
}

template <int BN, int KS>
llama_status launch_gemm_sk(int epi, const CUtensorMap& a, const CUtensorMap* w, const GemmParams& p, int grid,
                            cudaStream_t st, int kind) {
  if constexpr (KS == 2 && BN == 16) {
    if (p.cl_split > 0) {
      switch (epi) {
        case EPI_BF16: return launch_gemm_cl<BN, EPI_BF16>(a, w, p, grid, st, kind);
        case EPI_RESID_F32: return launch_gemm_cl<BN, EPI_RESID_F32>(a, w, p, grid, st, kind);
        case EPI_SWIGLU_BF16: return launch_gemm_cl<BN, EPI_SWIGLU_BF16>(a, w, p, grid, st, kind);
      }
      return LLAMA_ERR_INVALID_ARG;
    }
  }
  switch (epi) {
    case EPI_BF16: return launch_gemm_tc<BN, true, EPI_BF16, KS>(a, w, p, grid, st, kind);
    case EPI_RESID_F32: return launch_gemm_tc<BN, true, EPI_RESID_F32, KS>(a, w, p, grid, st, kind);
    case EPI_SWIGLU_BF16: return launch_gemm_tc<BN, true, EPI_SWIGLU_BF16, KS>(a, w, p, grid, st, kind);
    case EPI_F32: return launch_gemm_tc<BN, true, EPI_F32, KS>(a, w, p, grid, st, kind);
  }
  return LLAMA_ERR_INVALID_ARG;
}

// RoPE + KV append fused into the prefill QKV GEMM (EPI_QKV_ROPE_BF16).
struct RopeArgs {
  void* kc;
  void* vc;
  const float* tab;   // per-token cos/sin, written by the first RMSNorm
  int L, p0, nh, nkv, hd, cap, style;
};

// Tile-mode (prefill) GEMM: out = epi(act[M, K] · W^T), W given as segments.
// Each 256 x 256 output tile runs on a CTA pair: every CTA loads 128 activation
// rows and 128 weight rows per k-block.
llama_status gemm_prefill(cudaStream_t st, const void* act, int M, int K, const WSeg* segs, int nseg, int epi,
                          void* out, int ldo, const float* resid, int ldr, DevStatus* status, int kind,
                          const RopeArgs* rope = nullptr) {
  constexpr int BN = 256;
  GemmParams p{};
  p.K = K;
  p.num_kb = cdiv(K, 64);
  p.act_rows = M;
  p.m_tiles = cdiv(M, 256);
  p.nseg = nseg;
  p.out = out;
  p.ldo = ldo;
  p.resid = resid;
  p.ldr = ldr;
  p.status = status;
  p.limit_ns = g_wait_limit_ns.load();
  if (epi == EPI_QKV_ROPE_BF16) {
    if (rope == nullptr || (rope->hd != 64 && rope->hd != 128)) return LLAMA_ERR_INVALID_ARG;
    p.kc = rope->kc;
    p.vc = rope->vc;
    p.rope_tab = rope->tab;
    p.L = rope->L;
    p.p0 = rope->p0;
    p.nh = rope->nh;
    p.nkv = rope->nkv;
    p.hd = rope->hd;
    p.cap = rope->cap;
    p.rope_style = rope->style;
  }
  CUtensorMap ta, tw[3];
  std::memset(tw, 0, sizeof(tw));
  if (!make_map_2d(&ta, act, K, M, 128)) return LLAMA_ERR_CUDA;
  if (epi == EPI_SWIGLU_BF16) {
    // segs[0] = gate (w1), segs[1] = up (w3), both [ffn, K]; one tile = 128 gate + 128 up rows
    p.nseg = 2;
    p.seg_rows[0] = segs[0].rows;
    p.seg_tile0[0] = 0;
    p.n_tiles = cdiv(segs[0].rows, BN / 2);
    p.seg_tile0[1] = p.n_tiles;
    p.seg_tile0[2] = p.n_tiles;
    p.seg_tile0[3] = p.n_tiles;
    if (!make_map_2d(&tw[0], segs[0].ptr, K, segs[0].rows, BN / 2)) return LLAMA_ERR_CUDA;
    if (!make_map_2d(&tw[1], segs[1].ptr, K, segs[1].rows, BN / 2)) return LLAMA_ERR_CUDA;
    tw[2] = tw[1];
  } else {
    int t = 0;
    for (int s = 0; s < nseg; ++s) {
      p.seg_rows[s] = segs[s].rows;
      p.seg_col0[s] = segs[s].col0;
      p.seg_tile0[s] = t;
      t += cdiv(segs[s].rows, BN);
      if (!make_map_2d(&tw[s], segs[s].ptr, K, segs[s].rows, BN / 2)) return LLAMA_ERR_CUDA;
    }
    for (int s = nseg; s < 3; ++s) tw[s] = tw[0];
    for (int s = nseg; s < 4; ++s) p.seg_tile0[s] = t;
    p.n_tiles = t;
  }
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = 2 * std::min(tiles, num_sms() / 2);
  switch (epi) {
    case EPI_BF16:
      return launch_gemm_tc<BN, false, EPI_BF16>(ta, tw, p, grid, st, kind);
    case EPI_RESID_F32:
      return launch_gemm_tc<BN, false, EPI_RESID_F32>(ta, tw, p, grid, st, kind);
    case EPI_SWIGLU_BF16:
      return launch_gemm_tc<BN, false, EPI_SWIGLU_BF16>(ta, tw, p, grid, st, kind);
    case EPI_F32:
      return launch_gemm_tc<BN, false, EPI_F32>(ta, tw, p, grid, st, kind);
    case EPI_QKV_ROPE_BF16:
      return launch_gemm_tc<BN, false, EPI_QKV_ROPE_BF16>(ta, tw, p, grid, st, kind);
  }
  return LLAMA_ERR_INVALID_ARG;
}

// Stream-K parameters and tensor maps of one decode GEMM (bf16, swapped:
// weight rows fill the MMA's M, the M token rows are its N = BN) over at most
// `max_grid` CTAs; *grid_out = the CTAs that share its units.
llama_status prep_decode_gemm(const void* act, int M, int K, const WSeg* segs, int nseg, int epi, void* out,
                              int ldo, const float* resid, int ldr, SkScratch sk, DevStatus* status, int BN, int KS,
                              int max_grid, GemmParams& p, CUtensorMap& ta, CUtensorMap* tw, int* grid_out) {
  p = GemmParams{};
  p.K = K;
  p.num_kb = cdiv(K, 64 * KS);
  p.act_rows = M;
  p.m_tiles = 1;
  p.nseg = nseg;
  p.out = out;
  p.ldo = ldo;
  p.resid = resid;
  p.ldr = ldr;
  p.status = status;
  p.limit_ns = g_wait_limit_ns.load();
  p.partial = sk.partial;
  p.flags = sk.flags;
  p.early_trigger = early_trigger();
  std::memset(tw, 0, 3 * sizeof(CUtensorMap));
  if (!make_map_2d(&ta, act, K, M, BN)) return LLAMA_ERR_CUDA;
  int t = 0;
  if (epi == EPI_SWIGLU_BF16) {
    // a weight tile = 64 gate rows + the matching 64 up rows
    p.seg_rows[0] = segs[0].rows;
    t = cdiv(segs[0].rows, 64);
    for (int s = 0; s < 2; ++s)
      if (!make_map_2d(&tw[s], segs[s].ptr, K, segs[s].rows, 64)) return LLAMA_ERR_CUDA;
    tw[2] = tw[0];
  } else {
    for (int s = 0; s < nseg; ++s) {
      p.seg_rows[s] = segs[s].rows;
      p.seg_col0[s] = segs[s].col0;
      p.seg_tile0[s] = t;
      t += cdiv(segs[s].rows, 128);
      if (!make_map_2d(&tw[s], segs[s].ptr, K, segs[s].rows, 128)) return LLAMA_ERR_CUDA;
    }
    for (int s = nseg; s < 3; ++s) tw[s] = tw[0];
  }
  for (int s = (epi == EPI_SWIGLU_BF16 ? 1 : nseg); s < 4; ++s) p.seg_tile0[s] = t;
  p.n_tiles = t;
  p.units = (long long)p.n_tiles * p.num_kb;
  // no CTA may have an empty unit range: a tile's finisher waits on every CTA between
  const int grid = (int)std::min<long long>(max_grid, p.units);
  if ((p.units + 1) * (kMaxSkGrid + 1) >= (1LL << 32)) return LLAMA_ERR_UNSUPPORTED;  // 32-bit unit math
  p.sk_grid = grid;
  *grid_out = grid;
  return LLAMA_OK;
}

// Stream-K (decode) GEMM: out = epilogue(act[M, K] · W^T) with W as the MMA's
// A operand.  The CTA that ends a weight tile adds the other CTAs' pieces of
// it (published in `sk.partial` under `sk.flags`) and applies the epilogue.
llama_status gemm_decode(cudaStream_t st, const void* act, int M, int K, const WSeg* segs, int nseg, int epi,
                         void* out, int ldo, const float* resid, int ldr, SkScratch sk, DevStatus* status,
                         int kind, const NormFuse* norm = nullptr, const NormB* nb = nullptr,
                         bool ssq_out = false) {
  const int BN = swap_bn(M);
  const int KS = decode_ksub();
  GemmParams p;
  CUtensorMap ta, tw[3];
  int grid = 0;
  TRY(prep_decode_gemm(act, M, K, segs, nseg, epi, out, ldo, resid, ldr, sk, status, BN, KS,
                       std::min(num_sms(), kMaxSkGrid), p, ta, tw, &grid));
  if (norm != nullptr) {
    p.norm_g = norm->g;
    p.norm_out = norm->out;
    p.norm_eps = norm->eps;
    p.ssq = sk.ssq;
    p.norm_ctr = reinterpret_cast<unsigned*>(reinterpret_cast<uint8_t*>(sk.flags) - kWsFlagsOffset + kWsNormCtrOffset);
  }
  if (ssq_out) {
    // the sums of squares of the rows this GEMM finishes, for the next GEMM's RMSNorm
    if (epi != EPI_RESID_F32 || norm != nullptr || p.n_tiles > kMaxNormTiles) return LLAMA_ERR_INVALID_ARG;
    p.ssq = sk.ssq;
    p.write_ssq = 1;
  }
  if (const int cl = decode_cluster_split(p.n_tiles, p.num_kb, BN, KS, epi); cl > 0) {
    p.cl_split = cl;
    grid = p.n_tiles * cl;
    p.sk_grid = grid;
  }
  if (nb != nullptr) {
    // the B operand from RMSNorm(x): the cluster form only, 16-byte aligned rows
    if (p.cl_split == 0 || BN != 16 || (nb->ldx & 3) != 0 || !aligned16(nb->x) || !aligned16(nb->g) ||
        nb->dim != K)
      return LLAMA_ERR_INVALID_ARG;
    p.nb_x = nb->x;
    p.nb_ldx = nb->ldx;
    p.nb_g = nb->g;
    p.nb_ssq = nb->ssq;
    p.nb_tiles = nb->tiles;
    p.nb_dim = nb->dim;
    p.nb_eps = nb->eps;
    if (nb->h != nullptr && !aligned16(nb->h)) return LLAMA_ERR_INVALID_ARG;
    p.nb_h = nb->h;
  }
  if (KS == 2) {
    switch (BN) {
      case 16: return launch_gemm_sk<16, 2>(epi, ta, tw, p, grid, st, kind);
      case 32: return launch_gemm_sk<32, 2>(epi, ta, tw, p, grid, st, kind);
      case 64: return launch_gemm_sk<64, 2>(epi, ta, tw, p, grid, st, kind);
      default: return launch_gemm_sk<128, 2>(epi, ta, tw, p, grid, st, kind);
    }
  }
  switch (BN) {
    case 16: return launch_gemm_sk<16, 1>(epi, ta, tw, p, grid, st, kind);
    case 32: return launch_gemm_sk<32, 1>(epi, ta, tw, p, grid, st, kind);
    case 64: return launch_gemm_sk<64, 1>(epi, ta, tw, p, grid, st, kind);
    default: return launch_gemm_sk<128, 1>(epi, ta, tw, p, grid, st, kind);
  }
}

// Prefill-or-decode dispatch of one projection.
llama_status gemm_bf16(cudaStream_t st, bool decode, const void* act, int M, int K, const WSeg* segs, int nseg,
                       int epi, void* out, int ldo, const float* resid, int ldr, SkScratch sk,
                       DevStatus* status, int kind, const NormFuse* norm = nullptr, const NormB* nb = nullptr,
                       bool ssq_out = false) {
  if (decode && M <= kSwapMaxTokens)
    return gemm_decode(st, act, M, K, segs, nseg, epi, out, ldo, resid, ldr, sk, status, kind, norm, nb, ssq_out);
  if (nb != nullptr || ssq_out) return LLAMA_ERR_INVALID_ARG;
  return gemm_prefill(st, act, M, K, segs, nseg, epi, out, ldo, resid, ldr, status, kind);
}

// Whether a decode residual GEMM over M token rows and `dim` output columns
// takes the following RMSNorm into its own end.  Off unless LLAMA_FUSE_NORM=1:
// the grid-wide wait at the GEMM's end measured no faster than a stand-alone
// RMSNorm kernel behind a programmatic-dependent launch (13B-shaped layer at
// batch 16: 0.346 vs 0.344 ms per step; Phi-3-mini-shaped model at batch 8:
// 3.38 vs 3.29 ms).
// True when the decode GEMM over these weight segments takes the cluster form
// (the same choice gemm_decode makes).
bool decode_gemm_clustered(int M, int K, const WSeg* segs, int nseg, int epi) {
  if (M > kSwapMaxTokens) return false;
  const int KS = decode_ksub();
  int tiles = 0;
  if (epi == EPI_SWIGLU_BF16) {
    tiles = cdiv(segs[0].rows, 64);
  } else {
    for (int s = 0; s < nseg; ++s) tiles += cdiv(segs[s].rows, 128);
  }
  return decode_cluster_split(tiles, cdiv(K, 64 * KS), swap_bn(M), KS, epi) > 0;
}

// The decode RMSNorms inside the GEMMs that consume them (cluster form; the
// residual GEMM before leaves each row's sums of squares per column tile).
// LLAMA_NORM_IN_GEMM=0 keeps them as kernels of their own.
bool norm_in_gemm_enabled(const llama_dims& d, int M) {
  static const bool on = [] {
    const char* e = std::getenv("LLAMA_NORM_IN_GEMM");
    return !(e != nullptr && e[0] == '0');
  }();
  return on && d.dtype == LLAMA_BF16 && M <= 16 && d.dim % 8 == 0 && cdiv(d.dim, 128) <= kMaxNormTiles;
}

bool norm_fusable(const llama_dims& d, int M) {
  static const bool on = [] {
    const char* e = std::getenv("LLAMA_FUSE_NORM");
    return e != nullptr && e[0] == '1';
  }();
  return on && d.dtype == LLAMA_BF16 && M <= kSwapMaxTokens && cdiv(d.dim, 128) <= kMaxNormTiles;
}

// ------------------------------------------------------------------ 4-bit group-64 decode GEMMs

struct Q4Seg {
  llama_q4_weight w;
  int rows;
  int col0;
};

template <int BN, int EPI>
llama_status launch_gemm_q4(const CUtensorMap& a, const Q4Maps& maps, const GemmParams& p, int grid, cudaStream_t st,
                            int kind) {
  using C = Q4Cfg<BN>;
  TRY(ensure_smem_attr(reinterpret_cast<const void*>(gemm_q4_kernel<BN, EPI>), C::SMEM_BYTES));
  {
    TRACE(kind, st);
    CUDA_TRY(launch_k(gemm_q4_kernel<BN, EPI>, grid, Q4_THREADS, C::SMEM_BYTES, st, a, maps, p));
  }
  LAUNCH_CHECK();
  return LLAMA_OK;
}

template <int BN>
llama_status launch_gemm_q4_epi(int epi, const CUtensorMap& a, const Q4Maps& maps, const GemmParams& p, int grid,
                                cudaStream_t st, int kind) {
  switch (epi) {
    case EPI_BF16: return launch_gemm_q4<BN, EPI_BF16>(a, maps, p, grid, st, kind);
    case EPI_RESID_F32: return launch_gemm_q4<BN, EPI_RESID_F32>(a, maps, p, grid, st, kind);
    case EPI_SWIGLU_BF16: return launch_gemm_q4<BN, EPI_SWIGLU_BF16>(a, maps, p, grid, st, kind);
  }
  return LLAMA_ERR_INVALID_ARG;
}

// Decode GEMM with 4-bit weights: out = epilogue(act[M, K] . W^T), W given as
// up to three segments (or, for EPI_SWIGLU_BF16, gate = segs[0], up = segs[1]).
llama_status gemm_decode_q4(cudaStream_t st, const void* act, int M, int K, const Q4Seg* segs, int nseg, int epi,
                            void* out, int ldo, const float* resid, int ldr, SkScratch sk, DevStatus* status,
                            int kind, const NormFuse* norm = nullptr) {
  if (M > kSwapMaxTokens || K % 64 != 0) return LLAMA_ERR_UNSUPPORTED;
  const int BN = swap_bn(M);
  GemmParams p{};
  p.K = K;
  p.num_kb = cdiv(K, 64 * Q4_KG);   // units of four groups; groups past K read as zeros
  p.act_rows = M;
  p.m_tiles = 1;
  p.nseg = nseg;
  p.out = out;
  p.ldo = ldo;
  p.resid = resid;
  p.ldr = ldr;
  p.status = status;
  p.limit_ns = g_wait_limit_ns.load();
  p.partial = sk.partial;
  p.flags = sk.flags;
  p.early_trigger = early_trigger();
  if (norm != nullptr) {
    p.norm_g = norm->g;
    p.norm_out = norm->out;
    p.norm_eps = norm->eps;
    p.ssq = sk.ssq;
    p.norm_ctr = reinterpret_cast<unsigned*>(reinterpret_cast<uint8_t*>(sk.flags) - kWsFlagsOffset + kWsNormCtrOffset);
  }
  CUtensorMap ta;
  Q4Maps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (!make_map_2d(&ta, act, K, M, BN)) return LLAMA_ERR_CUDA;
  for (int s = 0; s < nseg; ++s) {
    const uint64_t rows = (uint64_t)segs[s].rows, groups = (uint64_t)K / 64;
    {
      const uint64_t dims[2] = {(uint64_t)K / 8, rows};
      const uint64_t strides[1] = {(uint64_t)K / 8 * 4};
      const uint32_t box[2] = {8 * Q4_KG, 64};
      if (!make_map_ex(&maps.codes[s], segs[s].w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, CU_TENSOR_MAP_SWIZZLE_NONE,
                       2, dims, strides, box))
        return LLAMA_ERR_CUDA;
    }
    const uint64_t dims[2] = {rows, groups};
    const uint64_t strides[1] = {rows * 2};
    const uint32_t box[2] = {64, Q4_KG};
    if (!make_map_ex(&maps.scales[s], segs[s].w.scales, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_NONE,
                     2, dims, strides, box) ||
        !make_map_ex(&maps.offsets[s], segs[s].w.offsets, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     CU_TENSOR_MAP_SWIZZLE_NONE, 2, dims, strides, box))
      return LLAMA_ERR_CUDA;
  }
  int t = 0;
  if (epi == EPI_SWIGLU_BF16) {
    p.seg_rows[0] = segs[0].rows;
    t = cdiv(segs[0].rows, 64);
    for (int s = 1; s < 4; ++s) p.seg_tile0[s] = t;
  } else {
    for (int s = 0; s < nseg; ++s) {
      p.seg_rows[s] = segs[s].rows;
      p.seg_col0[s] = segs[s].col0;
      p.seg_tile0[s] = t;
      t += cdiv(segs[s].rows, 128);
    }
    for (int s = nseg; s < 4; ++s) p.seg_tile0[s] = t;
  }
  p.n_tiles = t;
  p.units = (long long)p.n_tiles * p.num_kb;
  const int grid = (int)std::min<long long>(std::min(num_sms(), kMaxSkGrid), p.units);
  if ((p.units + 1) * (kMaxSkGrid + 1) >= (1LL << 32)) return LLAMA_ERR_UNSUPPORTED;
  p.sk_grid = grid;
  switch (BN) {
    case 16: return launch_gemm_q4_epi<16>(epi, ta, maps, p, grid, st, kind);
    case 32: return launch_gemm_q4_epi<32>(epi, ta, maps, p, grid, st, kind);
    case 64: return launch_gemm_q4_epi<64>(epi, ta, maps, p, grid, st, kind);
    default: return launch_gemm_q4_epi<128>(epi, ta, maps, p, grid, st, kind);
  }
}

// ------------------------------------------------------------------ attention launchers

// Ragged batch (tab != nullptr): L is the longest sequence's new tokens, Mtot
// the packed rows in all and T the most keys any sequence sees; the per-
// sequence values come from the device table.
// Which prefill-attention kernel runs: 1 = attn_prefill_kernel (two query
// tiles share each K/V tile, 128-key steps, one S buffer per tile), 2 =
// attn_prefill_k64_kernel (the same with 64-key steps and two S buffers per
// tile).  Default: 2 for head_dim below 128, 1 at 128.
// LLAMA_ATTN_FORM=pair | k64 takes one kernel for every shape.
int attn_prefill_form(int hd) {
  static const int forced = [] {
    const char* e = std::getenv("LLAMA_ATTN_FORM");
    if (e == nullptr) return 0;
    return std::strcmp(e, "pair") == 0 ? 1 : std::strcmp(e, "k64") == 0 ? 2 : 0;
  }();
  if (forced != 0) return forced;
  return hd < 128 ? 2 : 1;
}

llama_status attn_prefill_bf16(cudaStream_t st, const llama_dims& d, llama_kv_cache* kv, int B, int L, int p0,
                               const __nv_bfloat16* qkv, __nv_bfloat16* out, DevStatus* status,
                               const SeqTab* tab = nullptr, int Mtot = 0, int Tmax = 0) {
  const int form = attn_prefill_form(d.head_dim);
  auto* kernel = form == 2 ? attn_prefill_k64_kernel : attn_prefill_kernel;
  TRY(ensure_smem_attr(reinterpret_cast<const void*>(kernel), ATT_SMEM));
  const int hd = d.head_dim;
  const int qkvn = (d.n_heads + 2 * d.n_kv_heads) * hd;
  const int T = tab != nullptr ? Tmax : p0 + L;
  CUtensorMap tq, tk, tv;
  if (tab != nullptr) {
    // packed rows of all sequences
    const uint64_t dims[2] = {(uint64_t)qkvn, (uint64_t)Mtot};
    const uint64_t strides[1] = {(uint64_t)qkvn * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_map(&tq, qkv, 2, dims, strides, box)) return LLAMA_ERR_CUDA;
  } else {
    const uint64_t dims[3] = {(uint64_t)qkvn, (uint64_t)L, (uint64_t)B};
    const uint64_t strides[2] = {(uint64_t)qkvn * 2, (uint64_t)L * qkvn * 2};
    const uint32_t box[3] = {64, 128, 1};
    if (!make_map(&tq, qkv, 3, dims, strides, box)) return LLAMA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)hd, (uint64_t)T, (uint64_t)B * d.n_kv_heads};
    const uint64_t strides[2] = {(uint64_t)hd * 2, (uint64_t)kv->capacity * hd * 2};
    const uint32_t box[3] = {64, 128, 1};
    if (!make_map(&tk, kv->k, 3, dims, strides, box)) return LLAMA_ERR_CUDA;
    if (!make_map(&tv, kv->v, 3, dims, strides, box)) return LLAMA_ERR_CUDA;
  }
  AttnPrefillParams p{};
  p.L = L;
  p.p0 = p0;
  p.nh = d.n_heads;
  p.nkv = d.n_kv_heads;
  p.hd = hd;
  // GQA (group >= 2): a CTA takes two query heads of one KV group over 128
  // query rows, sharing every K/V tile; MHA: one head over 256 query rows
  p.head_pair = (d.n_heads / d.n_kv_heads) >= 2 ? 1 : 0;
  p.n_qblocks = cdiv(L, p.head_pair ? 128 : 256);
  p.scale_log2 = kLog2e / sqrtf((float)hd);
  p.out = out;
  p.status = status;
  p.limit_ns = g_wait_limit_ns.load();
  p.tab = tab;
  // heaviest query blocks dispatched first (see the kernel)
  dim3 grid(p.head_pair ? d.n_heads / 2 : d.n_heads, B, p.n_qblocks);
  TRACE(K_ATTN_PREFILL, st);
  CUDA_TRY(launch_k(kernel, grid, ATT_THREADS, ATT_SMEM, st, tq, tk, tv, p));
  LAUNCH_CHECK();
  return LLAMA_OK;
}

template <int HD, int G>
cudaError_t launch_attn_decode(const AttnDecodeParams& p, dim3 grid, cudaStream_t st, bool rope) {
  if (rope) return launch_k(attn_decode_kernel<HD, G, true>, grid, 128, 0, st, p);
  return launch_k(attn_decode_kernel<HD, G, false>, grid, 128, 0, st, p);
}

// K/V chunks in flight per CTA of the tensor-core decode attention
// (LLAMA_DECODE_MMA_STAGES=3 or 4, default 3): three 32 KB stages let two CTAs
// share an SM (70B-shaped decode, batch 64, cache 4096: attention 163 vs 177
// us, block 0.499 vs 0.513 ms with four).
int decode_mma_stages() {
  static const int n = [] {
    const char* e = std::getenv("LLAMA_DECODE_MMA_STAGES");
    return (e != nullptr && e[0] == '4') ? 4 : 3;
  }();
  return n;
}

template <int HD, int G, int ST, bool ROPE>
llama_status launch_attn_decode_mma_st(const CUtensorMap& tk, const CUtensorMap& tv, const AttnDecodeMmaParams& p,
                                       dim3 grid, cudaStream_t st) {
  using C = DecMmaCfg<HD, ST>;
  TRY(ensure_smem_attr(reinterpret_cast<const void*>(attn_decode_mma_kernel<HD, G, ST, ROPE>), C::SMEM));
  CUDA_TRY(launch_k(attn_decode_mma_kernel<HD, G, ST, ROPE>, grid, 32 * (ST + 1), C::SMEM, st, tk, tv, p));
  return LLAMA_OK;
}

template <int HD, int G>
llama_status launch_attn_decode_mma(const CUtensorMap& tk, const CUtensorMap& tv, const AttnDecodeMmaParams& p,
                                    dim3 grid, cudaStream_t st, bool rope) {
  if (decode_mma_stages() == 3)
    return rope ? launch_attn_decode_mma_st<HD, G, 3, true>(tk, tv, p, grid, st)
                : launch_attn_decode_mma_st<HD, G, 3, false>(tk, tv, p, grid, st);
  return rope ? launch_attn_decode_mma_st<HD, G, 4, true>(tk, tv, p, grid, st)
              : launch_attn_decode_mma_st<HD, G, 4, false>(tk, tv, p, grid, st);
}

// Decode attention for GQA groups of 4 or 8 on the tensor cores.
// Key splits of the tensor-core decode attention (and keys per split, whole
// 64-key chunks): one when the (sequence, KV head) grid covers every SM (two
// CTAs fit on one), else about two CTAs per SM.  Clamped to [min_splits, max_splits].
int mma_decode_splits(const llama_dims& d, int B, int T, int min_splits, int max_splits, int* kps_out) {
  const int base = B * d.n_kv_heads;
  int splits = base >= num_sms() ? 1 : cdiv(2 * num_sms(), base);
  splits = std::max(1, std::min(splits, std::min(kMaxAttnSplits, cdiv(T, 256))));
  if (forced_decode_splits() > 0) splits = std::min(forced_decode_splits(), std::min(kMaxAttnSplits, cdiv(T, DEC_CHUNK)));
  splits = std::max(std::min(min_splits, cdiv(T, DEC_CHUNK)), std::min(splits, max_splits));
  const int kps = cdiv(cdiv(T, splits), DEC_CHUNK) * DEC_CHUNK;
  if (kps_out != nullptr) *kps_out = kps;
  return cdiv(T, kps);
}

struct RopeFuse {
  float theta;
  int style;
};

llama_status attn_decode_mma(cudaStream_t st, const llama_dims& d, const void* kc, const void* vc, int capacity,
                             int B, int T, const __nv_bfloat16* qkv, int ld_qkv, __nv_bfloat16* out,
                             float* part_ml, float* part_o, DevStatus* status, int min_splits, int max_splits,
                             const SeqTab* tab, const RopeFuse* rope = nullptr) {
  const int hd = d.head_dim, grp = d.n_heads / d.n_kv_heads;
  CUtensorMap tk, tv;
  // a head_dim of 96 runs as 128: the second 64-dim box reads dims 64..95 and
  // the bounds fill 96..127 with zeros
  const uint64_t dims[3] = {(uint64_t)hd, (uint64_t)T, (uint64_t)B * d.n_kv_heads};
  const uint64_t strides[2] = {(uint64_t)hd * 2, (uint64_t)capacity * hd * 2};
  const uint32_t box[3] = {64, (uint32_t)DEC_CHUNK, 1};
  if (!make_map(&tk, kc, 3, dims, strides, box)) return LLAMA_ERR_CUDA;
  if (!make_map(&tv, vc, 3, dims, strides, box)) return LLAMA_ERR_CUDA;
  AttnDecodeMmaParams p{};
  p.qkv = qkv;
  p.ld_qkv = ld_qkv;
  p.hd = hd;
  p.T = T;
  p.nh = d.n_heads;
  p.nkv = d.n_kv_heads;
  p.scale_log2 = kLog2e / sqrtf((float)hd);
  p.part_ml = part_ml;
  p.part_o = part_o;
  p.out = out;
  p.status = status;
  p.limit_ns = g_wait_limit_ns.load();
  p.tab = tab;
  int kps = 0;
  const int splits = mma_decode_splits(d, B, T, min_splits, max_splits, &kps);
  if (rope != nullptr && splits != 1) return LLAMA_ERR_UNSUPPORTED;
  p.kc = reinterpret_cast<__nv_bfloat16*>(const_cast<void*>(kc));
  p.vc = reinterpret_cast<__nv_bfloat16*>(const_cast<void*>(vc));
  p.cap = capacity;
  p.theta = rope != nullptr ? rope->theta : 0.f;
  p.rope_style = rope != nullptr ? rope->style : 0;
  p.splits = splits;
  p.keys_per_split = kps;
  dim3 grid(splits, d.n_kv_heads, B);
  llama_status r = LLAMA_ERR_UNSUPPORTED;
  {
    TRACE(K_ATTN_DECODE, st);
#define DEC_MMA_CASE(HD_, G_) \
    if ((hd == HD_ || (HD_ == 128 && hd == 96)) && grp == G_) \
      r = launch_attn_decode_mma<HD_, G_>(tk, tv, p, grid, st, rope != nullptr);
    DEC_MMA_CASE(128, 8) else DEC_MMA_CASE(128, 4) else DEC_MMA_CASE(128, 2) else DEC_MMA_CASE(128, 1)
    else DEC_MMA_CASE(64, 8) else DEC_MMA_CASE(64, 4) else DEC_MMA_CASE(64, 2) else DEC_MMA_CASE(64, 1)
#undef DEC_MMA_CASE
  }
  if (r != LLAMA_OK) return r;
  LAUNCH_CHECK();
  if (splits > 1) {
    TRACE(K_ATTN_COMBINE, st);
    CUDA_TRY(launch_k(attn_decode_combine_kernel, dim3(d.n_heads, B), 128, 0, st, part_ml, part_o, out, d.n_heads, hd, splits,
                      early_trigger()));
  }
  LAUNCH_CHECK();
  return LLAMA_OK;
}

// Key splits of the CUDA-core decode attention (and keys per split, a multiple
// of 32).  One CTA per (sequence, KV head) when that alone fills 4 CTAs per SM,
// or fills every SM once and the cache is short (then there is no combine pass,
// which costs more than the extra loads in flight would save); otherwise split
// the keys for about 8 CTAs per SM, >= 64 keys per split (more, shorter splits
// keep more loads in flight).  Clamped to [min_splits, max_splits].
int simt_decode_splits(const llama_dims& d, int B, int T, int min_splits, int max_splits, int* kps_out) {
  const int base = B * d.n_kv_heads;
  int splits = (base >= 4 * num_sms() || (base >= num_sms() && T <= 2048)) ? 1 : cdiv(8 * num_sms(), base);
  splits = std::max(1, std::min(splits, std::min(kMaxAttnSplits, cdiv(T, 64))));
  if (forced_decode_splits() > 0) splits = std::min(forced_decode_splits(), std::min(kMaxAttnSplits, cdiv(T, 32)));
  splits = std::max(std::min(min_splits, cdiv(T, 32)), std::min(splits, max_splits));
  int kps = cdiv(T, splits);
  kps = cdiv(kps, 32) * 32;
  if (kps_out != nullptr) *kps_out = kps;
  return cdiv(T, kps);
}

// LLAMA_FUSE_ROPE=0 keeps RoPE + KV append a kernel of its own in decode.
bool rope_fuse_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("LLAMA_FUSE_ROPE");
    return !(e != nullptr && e[0] == '0');
  }();
  return on;
}

// Whether the decode attention over keys [0, T) does RoPE + KV append itself
// (attn_decode_bf16 with `rope`): either kernel with one key split, so that
// one CTA owns the new token's q heads and k/v row of its KV head.
bool decode_rope_fusable(const llama_dims& d, int B, int T, int min_splits = 1, int max_splits = kMaxAttnSplits) {
  if (!rope_fuse_enabled() || d.dtype != LLAMA_BF16) return false;
  if (use_decode_mma(d.head_dim, d.n_heads / d.n_kv_heads))
    return mma_decode_splits(d, B, T, min_splits, max_splits, nullptr) == 1;
  return simt_decode_splits(d, B, T, min_splits, max_splits, nullptr) == 1;
}

// Decode attention of one new token per sequence over keys [0, T).  Splits of
// the key range are chosen by a heuristic, clamped to [min_splits, max_splits].
// Ragged batch (tab != nullptr): T is the most keys any sequence sees;
// sequence b sees tab->p0[b] + 1.
// rope != nullptr (only where decode_rope_fusable holds): qkv holds the raw
// projections and the kernel does RoPE + KV append of the new token itself.
llama_status attn_decode_bf16(cudaStream_t st, const llama_dims& d, const void* kc, const void* vc, int capacity,
                              int B, int T, const __nv_bfloat16* qkv, int ld_qkv, __nv_bfloat16* out,
                              float* part_ml, float* part_o, DevStatus* status, int min_splits = 1,
                              int max_splits = kMaxAttnSplits, const SeqTab* tab = nullptr,
                              const RopeFuse* rope = nullptr) {
  const int hd = d.head_dim, grp = d.n_heads / d.n_kv_heads;
  if (use_decode_mma(hd, grp))
    return attn_decode_mma(st, d, kc, vc, capacity, B, T, qkv, ld_qkv, out, part_ml, part_o, status, min_splits,
                           max_splits, tab, rope);
  AttnDecodeParams p{};
  p.qkv = qkv;
  p.ld_qkv = ld_qkv;
  p.kc = reinterpret_cast<const __nv_bfloat16*>(kc);
  p.vc = reinterpret_cast<const __nv_bfloat16*>(vc);
  p.cap = capacity;
  p.T = T;
  p.nh = d.n_heads;
  p.nkv = d.n_kv_heads;
  p.scale_log2 = kLog2e / sqrtf((float)hd);
  p.part_ml = part_ml;
  p.part_o = part_o;
  p.out = out;
  p.tab = tab;
  int kps = 0;
  const int splits = simt_decode_splits(d, B, T, min_splits, max_splits, &kps);
  if (rope != nullptr && splits != 1) return LLAMA_ERR_UNSUPPORTED;
  p.splits = splits;
  p.keys_per_split = kps;
  p.theta = rope != nullptr ? rope->theta : 0.f;
  p.rope_style = rope != nullptr ? rope->style : 0;
  dim3 grid(splits, d.n_kv_heads, B);
  {
  TRACE(K_ATTN_DECODE, st);
#define DEC_CASE(HD_, G_) \
  if (hd == HD_ && grp == G_) CUDA_TRY((launch_attn_decode<HD_, G_>(p, grid, st, rope != nullptr)));
  DEC_CASE(64, 1) DEC_CASE(64, 2) DEC_CASE(64, 4) DEC_CASE(64, 8)
  DEC_CASE(96, 1) DEC_CASE(96, 2) DEC_CASE(96, 4) DEC_CASE(96, 8)
  DEC_CASE(128, 1) DEC_CASE(128, 2) DEC_CASE(128, 4) DEC_CASE(128, 8)
#undef DEC_CASE
  }
  LAUNCH_CHECK();
  if (splits > 1) {
    TRACE(K_ATTN_COMBINE, st);
    CUDA_TRY(launch_k(attn_decode_combine_kernel, dim3(d.n_heads, B), 128, 0, st, part_ml, part_o, out, d.n_heads, hd, splits,
                      early_trigger()));
    LAUNCH_CHECK();
  }
  return LLAMA_OK;
}

// ------------------------------------------------------------------ persistent decode block

// Whether a decode step of B token rows runs as one persistent kernel
// (decode_layer_kernel): only with LLAMA_DECODE_LAYER=1, and for bf16, B <= 16,
// head_dim 64 / 96 / 128, GQA group 1 or 2, when the attention's (sequence, KV
// head) units fit the CTAs' two groups in one round or the cache is short (the
// kernel runs one key split per unit).  Off by default: measured slower than
// the kernel-per-step chain (Phi-3-mini-shaped block, batch 8, cache 512:
// 0.125 vs 0.097 ms; 13B-shaped, batch 16: 0.216 vs 0.172 ms).
bool decode_layer_fusable(const llama_dims& d, int B, int T) {
  static const bool on = [] {
    const char* e = std::getenv("LLAMA_DECODE_LAYER");
    return e != nullptr && e[0] == '1';
  }();
  const int hd = d.head_dim, grp = d.n_heads / d.n_kv_heads;
  if (!on || d.dtype != LLAMA_BF16 || B < 1 || B > DL_BN) return false;
  if (!(hd == 64 || hd == 96 || hd == 128) || !(grp == 1 || grp == 2)) return false;
  if (decode_attn_forced() == 1) return false;   // forced tensor-core decode attention (LLAMA_DECODE_ATTN=mma)
  if (d.dim % 64 != 0 || cdiv(d.dim, 128) > kMaxNormTiles || num_sms() > kMaxSkGrid) return false;
  return B * d.n_kv_heads <= 2 * num_sms() || T <= 2048;
}

// LLAMA_DL_PREFETCH=1: the persistent decode block's producer also prefetches
// upcoming weight tiles and the attention's cache rows into L2.
bool dl_l2_prefetch() {
  static const bool on = [] {
    const char* e = std::getenv("LLAMA_DL_PREFETCH");
    return e != nullptr && e[0] == '1';
  }();
  return on;
}

template <int HD, int G>
llama_status launch_decode_layer(const DecLayerParams& P, cudaStream_t st) {
  using S = DecLayerSmem<HD, G>;
  TRY(ensure_smem_attr(reinterpret_cast<const void*>(decode_layer_kernel<HD, G>), S::BYTES));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(num_sms());   // one CTA per SM, all resident (cooperative launch)
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = S::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    TRACE(K_DECODE_LAYER, st);
    CUDA_TRY(cudaLaunchKernelEx(&cfg, decode_layer_kernel<HD, G>, P));
  }
  LAUNCH_CHECK();
  return LLAMA_OK;
}

// One decode step of a block (bf16, B token rows at cache length p0) as one
// persistent kernel; the caller has checked decode_layer_fusable.
llama_status run_decode_layer(const llama_dims& d, const llama_layer_weights& w, llama_kv_cache* kv, int B,
                              const float* x_in, float* x_out, uint8_t* ws, const WsLayout& lay, cudaStream_t st,
                              const WSeg* segs, int nseg) {
  using bf = __nv_bfloat16;
  const int nh = d.n_heads, nkv = d.n_kv_heads, hd = d.head_dim;
  const int qkvn = (nh + 2 * nkv) * hd;
  const int p0 = kv->length, T = p0 + 1;
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  bf* qkv = reinterpret_cast<bf*>(ws + lay.qkv);
  bf* h = reinterpret_cast<bf*>(ws + lay.h);
  bf* att = reinterpret_cast<bf*>(ws + lay.attn);
  bf* mb = reinterpret_cast<bf*>(ws + lay.mbuf);
  const SkScratch sk{reinterpret_cast<float*>(ws + lay.partial), reinterpret_cast<unsigned*>(ws + lay.sk_flags),
                     reinterpret_cast<float*>(ws + lay.ssq)};
  const int G = num_sms();
  DecLayerParams P;
  std::memset(&P, 0, sizeof(P));
  int grid = 0;
  TRY(prep_decode_gemm(h, B, d.dim, segs, nseg, EPI_BF16, qkv, qkvn, nullptr, 0, sk, status, DL_BN, DL_KS, G,
                       P.g[DL_QKV], P.act[DL_QKV], P.w[DL_QKV], &grid));
  const WSeg so{w.wo, d.dim, 0};
  TRY(prep_decode_gemm(att, B, nh * hd, &so, 1, EPI_RESID_F32, x_out, d.dim, x_in, d.dim, sk, status, DL_BN, DL_KS,
                       G, P.g[DL_O], P.act[DL_O], P.w[DL_O], &grid));
  P.g[DL_O].norm_g = w.ffn_norm;   // per-tile sums of squares for RMSNorm-2 (no counter)
  P.g[DL_O].ssq = sk.ssq;
  const WSeg sg[2] = {{w.w1, d.ffn_dim, 0}, {w.w3, d.ffn_dim, 0}};
  TRY(prep_decode_gemm(h, B, d.dim, sg, 2, EPI_SWIGLU_BF16, mb, d.ffn_dim, nullptr, 0, sk, status, DL_BN, DL_KS, G,
                       P.g[DL_GU], P.act[DL_GU], P.w[DL_GU], &grid));
  const WSeg sd{w.w2, d.dim, 0};
  TRY(prep_decode_gemm(mb, B, d.ffn_dim, &sd, 1, EPI_RESID_F32, x_out, d.dim, x_out, d.dim, sk, status, DL_BN,
                       DL_KS, G, P.g[DL_DOWN], P.act[DL_DOWN], P.w[DL_DOWN], &grid));
  AttnDecodeParams& a = P.attn;
  a.qkv = qkv;
  a.ld_qkv = qkvn;
  a.kc = reinterpret_cast<const bf*>(kv->k);
  a.vc = reinterpret_cast<const bf*>(kv->v);
  a.cap = kv->capacity;
  a.T = T;
  a.nh = nh;
  a.nkv = nkv;
  a.splits = 1;
  a.keys_per_split = cdiv(T, 32) * 32;
  a.scale_log2 = kLog2e / sqrtf((float)hd);
  a.out = att;
  a.theta = d.rope_theta;
  a.rope_style = d.rope_style;
  P.x_in = x_in;
  P.x_out = x_out;
  P.attn_norm = w.attn_norm;
  P.ffn_norm = w.ffn_norm;
  P.h = h;
  P.ssq = sk.ssq;
  P.slots = sk.ssq + (size_t)kMaxNormTiles * DL_BN;
  P.bar = reinterpret_cast<unsigned*>(ws + kWsGridBarOffset);
  P.status = status;
  P.limit_ns = g_wait_limit_ns.load();
  P.eps = d.eps;
  P.dim = d.dim;
  P.B = B;
  P.l2_prefetch = dl_l2_prefetch();
  const int grp = nh / nkv;
#define DL_CASE(HD_, G_) \
  if (hd == HD_ && grp == G_) return launch_decode_layer<HD_, G_>(P, st);
  DL_CASE(64, 1) DL_CASE(64, 2) DL_CASE(96, 1) DL_CASE(96, 2) DL_CASE(128, 1) DL_CASE(128, 2)
#undef DL_CASE
  return LLAMA_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ one block

llama_status check_layer_call(const llama_dims* dims, const llama_layer_weights* w, llama_kv_cache* kv, int B,
                              int L, const float* x_in, float* x_out, void* ws, size_t ws_bytes, int vocab) {
  TRY(check_dims(dims));
  TRY(check_weights(w));
  if (kv == nullptr || x_in == nullptr || x_out == nullptr || ws == nullptr) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || L <= 0) return LLAMA_ERR_INVALID_ARG;
  if (!same_dims(*dims, kv->dims) || B != kv->batch) return LLAMA_ERR_INVALID_ARG;
  if (!kv->lens.empty()) return LLAMA_ERR_INVALID_ARG;   // per-sequence lengths: llama_layer_forward_ragged
  if (!aligned16(x_in) || !aligned16(x_out) || !aligned16(ws)) return LLAMA_ERR_ALIGNMENT;
  const size_t xb = (size_t)B * L * dims->dim * 4;
  if (overlap(x_in, xb, x_out, xb)) return LLAMA_ERR_INVALID_ARG;
  if ((long long)kv->length + L > kv->capacity) return LLAMA_ERR_CACHE_FULL;
  if (ws_bytes < plan_ws(*dims, B, L, vocab).total) return LLAMA_ERR_WORKSPACE_TOO_SMALL;
  return LLAMA_OK;
}

// Enqueue one block.  `decode` selects the one-token-per-sequence kernels.
// Decode with the fused norms (norm_fusable): RMSNorm-2 runs at the end of the
// o_proj GEMM; `next_norm` (if any) is the RMSNorm that follows this block --
// the next block's first one, or the model's final one -- run at the end of
// the down GEMM into `next_out`; `h_ready`: this block's RMSNorm-1 output is
// already in the workspace (the previous block's down GEMM wrote it).
// x_ssq_ready: the workspace's sums of squares hold x_in's rows (written by
// the previous block's down GEMM); ssq_next: this block's down GEMM writes
// them for the next block.
llama_status run_layer(const llama_dims& d, const llama_layer_weights& w, llama_kv_cache* kv, int B, int L,
                       const float* x_in, float* x_out, uint8_t* ws, const WsLayout& lay, cudaStream_t st,
                       const float* next_norm = nullptr, void* next_out = nullptr, bool h_ready = false,
                       bool x_ssq_ready = false, bool ssq_next = false) {
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  const int M = B * L;
  const int nh = d.n_heads, nkv = d.n_kv_heads, hd = d.head_dim;
  const int qkvn = (nh + 2 * nkv) * hd;
  const int p0 = kv->length;
  const bool decode = (L == 1);
  const int rows_per_block = 256 / 32;
  if (d.dtype == LLAMA_BF16) {
    using bf = __nv_bfloat16;
    bf* qkv = reinterpret_cast<bf*>(ws + lay.qkv);
    bf* h = reinterpret_cast<bf*>(ws + lay.h);
    bf* att = reinterpret_cast<bf*>(ws + lay.attn);
    bf* mb = reinterpret_cast<bf*>(ws + lay.mbuf);
    // prefill with head_dim 64 / 128: RoPE and the cache append run in the QKV GEMM's epilogue
    const bool fuse_rope = !decode && (hd == 64 || hd == 128);
    float* rtab = reinterpret_cast<float*>(ws + lay.rope_tab);
    const SkScratch part{reinterpret_cast<float*>(ws + lay.partial), reinterpret_cast<unsigned*>(ws + lay.sk_flags),
                         reinterpret_cast<float*>(ws + lay.ssq)};
    const bool fuse_norm = decode && norm_fusable(d, M);
    // a QKV projection reads one weight buffer when q, k and v sit back to back
    const size_t rb = (size_t)d.dim * 2;  // bytes per weight row
    WSeg segs[3];
    int nseg;
    if (w.wk == (const uint8_t*)w.wq + (size_t)nh * hd * rb && w.wv == (const uint8_t*)w.wk + (size_t)nkv * hd * rb) {
      segs[0] = {w.wq, qkvn, 0};
      nseg = 1;
    } else {
      segs[0] = {w.wq, nh * hd, 0};
      segs[1] = {w.wk, nkv * hd, nh * hd};
      segs[2] = {w.wv, nkv * hd, (nh + nkv) * hd};
      nseg = 3;
    }
    // decode at batch <= 16: the whole block in one persistent kernel
    if (decode && !fuse_norm && decode_layer_fusable(d, B, p0 + 1)) {
      TRY(run_decode_layer(d, w, kv, B, x_in, x_out, ws, lay, st, segs, nseg));
      kv->length = p0 + L;
      return LLAMA_OK;
    }
    // RMSNorms inside the consuming GEMMs (cluster form): RMSNorm-1 when the
    // previous block left x_in's sums of squares, RMSNorm-2 from o_proj's
    const bool nig = decode && !fuse_norm && norm_in_gemm_enabled(d, M);
    const bool nig1 = nig && x_ssq_ready && decode_gemm_clustered(M, d.dim, segs, nseg, EPI_BF16);
    WSeg sg[2] = {{w.w1, d.ffn_dim, 0}, {w.w3, d.ffn_dim, 0}};
    const bool nig2 = nig && decode_gemm_clustered(M, d.dim, sg, 2, EPI_SWIGLU_BF16);
    const int ssq_tiles = cdiv(d.dim, 128);
    const NormB nb1{x_in, d.dim, w.attn_norm, part.ssq, ssq_tiles, d.dim, d.eps, h};
    const NormB nb2{x_out, d.dim, w.ffn_norm, part.ssq, ssq_tiles, d.dim, d.eps, h};
    // a2: RMSNorm-1 -> h (bf16)
    if (!(fuse_norm && h_ready) && !nig1) {
      TRACE(K_RMSNORM, st);
      // with RoPE fused into the QKV GEMM, it also writes each token's cos/sin row
      const RopeTab rt{fuse_rope ? rtab : nullptr, hd, L, p0, d.rope_theta, early_trigger()};
      CUDA_TRY(launch_k(rmsnorm_kernel<bf>, M, rmsnorm_threads(d.dim), 0, st, x_in, d.dim, w.attn_norm, h, M, d.dim,
                        d.eps, rt));
      LAUNCH_CHECK();
    }
    // a3: QKV projection
    const bool rope_in_attn = decode && decode_rope_fusable(d, B, p0 + 1);
    const RopeFuse rf{d.rope_theta, d.rope_style};
    if (fuse_rope) {
      // a3 + a4 in one kernel: rotated q -> qkv, rotated k and v -> the cache
      const RopeArgs ra{kv->k, kv->v, rtab, L, p0, nh, nkv, hd, kv->capacity, d.rope_style};
      TRY(gemm_prefill(st, h, M, d.dim, segs, nseg, EPI_QKV_ROPE_BF16, qkv, qkvn, nullptr, 0, status, K_GEMM_QKV,
                       &ra));
    } else {
      TRY(gemm_bf16(st, decode, h, M, d.dim, segs, nseg, EPI_BF16, qkv, qkvn, nullptr, 0, part, status, K_GEMM_QKV,
                    nullptr, nig1 ? &nb1 : nullptr));
      // a4: RoPE + KV append (decode with one key split: inside the attention kernel)
      if (!rope_in_attn) {
        TRACE(K_ROPE_APPEND, st);
        CUDA_TRY(launch_k(rope_append_kernel<bf>, M, 256, 0, st, qkv, reinterpret_cast<bf*>(kv->k),
                          reinterpret_cast<bf*>(kv->v), L, p0, nh, nkv, hd, kv->capacity, d.rope_theta,
                          d.rope_style, static_cast<const SeqTab*>(nullptr)));
        LAUNCH_CHECK();
      }
    }
    // a5 / a6: attention
    if (decode) {
      TRY(attn_decode_bf16(st, d, kv->k, kv->v, kv->capacity, B, p0 + 1, qkv, qkvn, att,
                           reinterpret_cast<float*>(ws + lay.att_ml), reinterpret_cast<float*>(ws + lay.att_o),
                           status, 1, kMaxAttnSplits, nullptr, rope_in_attn ? &rf : nullptr));
    } else {
      TRY(attn_prefill_bf16(st, d, kv, B, L, p0, qkv, att, status));
    }
    // a7: o_proj + residual -> x_out holds x_mid (decode: RMSNorm-2 at its end)
    WSeg so{w.wo, d.dim, 0};
    const NormFuse n2{w.ffn_norm, h, d.eps};
    TRY(gemm_bf16(st, decode, att, M, nh * hd, &so, 1, EPI_RESID_F32, x_out, d.dim, x_in, d.dim, part, status,
                  K_GEMM_O, fuse_norm ? &n2 : nullptr, nullptr, nig2));
    // a8: RMSNorm-2 + gate_up + SiLU·mul
    if (!fuse_norm && !nig2) {
      TRACE(K_RMSNORM, st);
      CUDA_TRY(launch_k(rmsnorm_kernel<bf>, M, rmsnorm_threads(d.dim), 0, st, x_out, d.dim, w.ffn_norm, h, M, d.dim,
                        d.eps, RopeTab{nullptr, 0, 0, 0, 0.f, early_trigger()}));
      LAUNCH_CHECK();
    }
    TRY(gemm_bf16(st, decode, h, M, d.dim, sg, 2, EPI_SWIGLU_BF16, mb, d.ffn_dim, nullptr, 0, part, status,
                  K_GEMM_GATE_UP, nullptr, nig2 ? &nb2 : nullptr));
    // a9: down + residual (in place on x_out); decode: the next RMSNorm at its end
    WSeg sd{w.w2, d.dim, 0};
    const NormFuse nn{next_norm, next_out, d.eps};
    TRY(gemm_bf16(st, decode, mb, M, d.ffn_dim, &sd, 1, EPI_RESID_F32, x_out, d.dim, x_out, d.dim, part, status,
                  K_GEMM_DOWN, (fuse_norm && next_norm != nullptr) ? &nn : nullptr, nullptr, nig && ssq_next));
  } else {
    float* qkv = reinterpret_cast<float*>(ws + lay.qkv);
    float* h = reinterpret_cast<float*>(ws + lay.h);
    float* att = reinterpret_cast<float*>(ws + lay.attn);
    float* mb = reinterpret_cast<float*>(ws + lay.mbuf);
    const float* wq = static_cast<const float*>(w.wq);
    const float* wk = static_cast<const float*>(w.wk);
    const float* wv = static_cast<const float*>(w.wv);
    auto grid_for = [](int M_, int N_) { return dim3(cdiv(N_, 64), cdiv(M_, 64)); };
    {
      TRACE(K_RMSNORM, st);
      rmsnorm_kernel<float><<<M, rmsnorm_threads(d.dim), 0, st>>>(x_in, d.dim, w.attn_norm, h, M, d.dim, d.eps,
                                                                   RopeTab{});
    }
    {
      TRACE(K_GEMM_F32, st);
      gemm_f32_kernel<F32_STORE><<<grid_for(M, nh * hd), 256, 0, st>>>(h, d.dim, wq, nullptr, d.dim, M, nh * hd,
                                                                        d.dim, qkv, qkvn, nullptr, 0);
    }
    {
      TRACE(K_GEMM_F32, st);
      gemm_f32_kernel<F32_STORE><<<grid_for(M, nkv * hd), 256, 0, st>>>(h, d.dim, wk, nullptr, d.dim, M, nkv * hd,
                                                                         d.dim, qkv + nh * hd, qkvn, nullptr, 0);
    }
    {
      TRACE(K_GEMM_F32, st);
      gemm_f32_kernel<F32_STORE><<<grid_for(M, nkv * hd), 256, 0, st>>>(
          h, d.dim, wv, nullptr, d.dim, M, nkv * hd, d.dim, qkv + (nh + nkv) * hd, qkvn, nullptr, 0);
    }
    LAUNCH_CHECK();
    {
      TRACE(K_ROPE_APPEND, st);
      rope_append_kernel<float><<<M, 256, 0, st>>>(qkv, static_cast<float*>(kv->k), static_cast<float*>(kv->v), L,
                                                    p0, nh, nkv, hd, kv->capacity, d.rope_theta, d.rope_style,
                                                    nullptr);
    }
    LAUNCH_CHECK();
    const int Tmax = p0 + L;
    const size_t smem = (size_t)Tmax * 4;
    if (smem > 200 * 1024) return LLAMA_ERR_UNSUPPORTED;
    if (smem > 48 * 1024) TRY(ensure_smem_attr(reinterpret_cast<const void*>(attn_f32_kernel), 200 * 1024));
    {
      TRACE(K_ATTN_F32, st);
      attn_f32_kernel<<<dim3(L, nh, B), 128, smem, st>>>(qkv, qkvn, static_cast<const float*>(kv->k),
                                                         static_cast<const float*>(kv->v), att, L, p0, nh, nkv, hd,
                                                         kv->capacity);
    }
    LAUNCH_CHECK();
    {
      TRACE(K_GEMM_F32, st);
      gemm_f32_kernel<F32_RESID><<<grid_for(M, d.dim), 256, 0, st>>>(att, nh * hd, static_cast<const float*>(w.wo),
                                                                     nullptr, nh * hd, M, d.dim, nh * hd, x_out,
                                                                     d.dim, x_in, d.dim);
    }
    LAUNCH_CHECK();
    {
      TRACE(K_RMSNORM, st);
      rmsnorm_kernel<float><<<M, rmsnorm_threads(d.dim), 0, st>>>(x_out, d.dim, w.ffn_norm, h, M, d.dim, d.eps,
                                                                    RopeTab{});
    }
    {
      TRACE(K_GEMM_F32, st);
      gemm_f32_kernel<F32_SWIGLU><<<grid_for(M, d.ffn_dim), 256, 0, st>>>(
          h, d.dim, static_cast<const float*>(w.w1), static_cast<const float*>(w.w3), d.dim, M, d.ffn_dim, d.dim,
          mb, d.ffn_dim, nullptr, 0);
    }
    {
      TRACE(K_GEMM_F32, st);
      gemm_f32_kernel<F32_RESID><<<grid_for(M, d.dim), 256, 0, st>>>(mb, d.ffn_dim, static_cast<const float*>(w.w2),
                                                                     nullptr, d.ffn_dim, M, d.dim, d.ffn_dim, x_out,
                                                                     d.dim, x_out, d.dim);
    }
    LAUNCH_CHECK();
  }
  kv->length = p0 + L;
  return LLAMA_OK;
}

// ------------------------------------------------------------------ one block, ragged batch

// Enqueue one block over a ragged batch: sequence b brings n_new[b] >= 1 new
// tokens, packed in sequence order in x_in, at positions from its own cache
// length on.  Decode rows and prefill chunks may be mixed: with every
// n_new[b] == 1 the split-KV decode attention runs, otherwise the flash
// attention in its varlen form (a one-token sequence is a one-row query block).
llama_status run_layer_ragged(const llama_dims& d, const llama_layer_weights& w, llama_kv_cache* kv, int B,
                              const int32_t* n_new, const float* x_in, float* x_out, uint8_t* ws,
                              const WsLayout& lay, cudaStream_t st) {
  using bf = __nv_bfloat16;
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  const int nh = d.n_heads, nkv = d.n_kv_heads, hd = d.head_dim;
  const int qkvn = (nh + 2 * nkv) * hd;
  SeqTab tab{};
  tab.n = B;
  int M = 0, maxL = 0, Tmax = 0;
  bool all_one = true;
  for (int b = 0; b < B; ++b) {
    const int p0 = kv->lens.empty() ? kv->length : kv->lens[b];
    tab.start[b] = M;
    tab.len[b] = n_new[b];
    tab.p0[b] = p0;
    M += n_new[b];
    maxL = std::max(maxL, n_new[b]);
    Tmax = std::max(Tmax, p0 + n_new[b]);
    all_one = all_one && n_new[b] == 1;
  }
  SeqTab* dtab = reinterpret_cast<SeqTab*>(ws + lay.seqtab);
  {
    TRACE(K_SEQTAB, st);
    CUDA_TRY(launch_k(seqtab_kernel, 1, 128, 0, st, tab, dtab));
  }
  LAUNCH_CHECK();
  const bool sk = M <= kSwapMaxTokens;   // few token rows: the swapped stream-K GEMMs
  bf* qkv = reinterpret_cast<bf*>(ws + lay.qkv);
  bf* h = reinterpret_cast<bf*>(ws + lay.h);
  bf* att = reinterpret_cast<bf*>(ws + lay.attn);
  bf* mb = reinterpret_cast<bf*>(ws + lay.mbuf);
  const SkScratch part{reinterpret_cast<float*>(ws + lay.partial), reinterpret_cast<unsigned*>(ws + lay.sk_flags),
                         reinterpret_cast<float*>(ws + lay.ssq)};
  {
    TRACE(K_RMSNORM, st);
    CUDA_TRY(launch_k(rmsnorm_kernel<bf>, M, rmsnorm_threads(d.dim), 0, st, x_in, d.dim, w.attn_norm, h, M, d.dim,
                      d.eps, RopeTab{nullptr, 0, 0, 0, 0.f, early_trigger()}));
  }
  LAUNCH_CHECK();
  const size_t rb = (size_t)d.dim * 2;
  WSeg segs[3];
  int nseg;
  if (w.wk == (const uint8_t*)w.wq + (size_t)nh * hd * rb && w.wv == (const uint8_t*)w.wk + (size_t)nkv * hd * rb) {
    segs[0] = {w.wq, qkvn, 0};
    nseg = 1;
  } else {
    segs[0] = {w.wq, nh * hd, 0};
    segs[1] = {w.wk, nkv * hd, nh * hd};
    segs[2] = {w.wv, nkv * hd, (nh + nkv) * hd};
    nseg = 3;
  }
  TRY(gemm_bf16(st, sk, h, M, d.dim, segs, nseg, EPI_BF16, qkv, qkvn, nullptr, 0, part, status, K_GEMM_QKV));
  // one new token per sequence and one key split: RoPE + KV append inside the attention kernel
  const bool rope_in_attn = all_one && decode_rope_fusable(d, B, Tmax);
  const RopeFuse rf{d.rope_theta, d.rope_style};
  if (!rope_in_attn) {
    TRACE(K_ROPE_APPEND, st);
    CUDA_TRY(launch_k(rope_append_kernel<bf>, M, 256, 0, st, qkv, reinterpret_cast<bf*>(kv->k),
                      reinterpret_cast<bf*>(kv->v), 1, 0, nh, nkv, hd, kv->capacity, d.rope_theta, d.rope_style,
                      static_cast<const SeqTab*>(dtab)));
    LAUNCH_CHECK();
  }
  if (all_one) {
    TRY(attn_decode_bf16(st, d, kv->k, kv->v, kv->capacity, B, Tmax, qkv, qkvn, att,
                         reinterpret_cast<float*>(ws + lay.att_ml), reinterpret_cast<float*>(ws + lay.att_o), status,
                         1, kMaxAttnSplits, dtab, rope_in_attn ? &rf : nullptr));
  } else {
    TRY(attn_prefill_bf16(st, d, kv, B, maxL, 0, qkv, att, status, dtab, M, Tmax));
  }
  WSeg so{w.wo, d.dim, 0};
  TRY(gemm_bf16(st, sk, att, M, nh * hd, &so, 1, EPI_RESID_F32, x_out, d.dim, x_in, d.dim, part, status, K_GEMM_O));
  {
    TRACE(K_RMSNORM, st);
    CUDA_TRY(launch_k(rmsnorm_kernel<bf>, M, rmsnorm_threads(d.dim), 0, st, x_out, d.dim, w.ffn_norm, h, M, d.dim,
                      d.eps, RopeTab{nullptr, 0, 0, 0, 0.f, early_trigger()}));
  }
  LAUNCH_CHECK();
  WSeg sg[2] = {{w.w1, d.ffn_dim, 0}, {w.w3, d.ffn_dim, 0}};
  TRY(gemm_bf16(st, sk, h, M, d.dim, sg, 2, EPI_SWIGLU_BF16, mb, d.ffn_dim, nullptr, 0, part, status,
                K_GEMM_GATE_UP));
  WSeg sd{w.w2, d.dim, 0};
  TRY(gemm_bf16(st, sk, mb, M, d.ffn_dim, &sd, 1, EPI_RESID_F32, x_out, d.dim, x_out, d.dim, part, status,
                K_GEMM_DOWN));
  // every sequence's length advances by its new tokens
  std::vector<int32_t> lens(B);
  for (int b = 0; b < B; ++b) lens[b] = tab.p0[b] + n_new[b];
  bool same = true;
  for (int b = 1; b < B; ++b) same = same && lens[b] == lens[0];
  if (same) {
    kv->length = lens[0];
    kv->lens.clear();
  } else {
    kv->length = -2;
    kv->lens = std::move(lens);
  }
  return LLAMA_OK;
}

// ------------------------------------------------------------------ one block, 4-bit weights (decode)

llama_status check_q4(const llama_q4_weight& w) {
  if (w.codes == nullptr || w.scales == nullptr || w.offsets == nullptr) return LLAMA_ERR_INVALID_ARG;
  if (!aligned16(w.codes) || !aligned16(w.scales) || !aligned16(w.offsets)) return LLAMA_ERR_ALIGNMENT;
  return LLAMA_OK;
}

llama_status check_layer_q4(const llama_dims* d, const llama_layer_weights_q4* w) {
  TRY(check_dims(d));
  if (w == nullptr || w->attn_norm == nullptr || w->ffn_norm == nullptr) return LLAMA_ERR_INVALID_ARG;
  if (!aligned16(w->attn_norm) || !aligned16(w->ffn_norm)) return LLAMA_ERR_ALIGNMENT;
  for (const llama_q4_weight* q : {&w->wq, &w->wk, &w->wv, &w->wo, &w->w1, &w->w3, &w->w2}) TRY(check_q4(*q));
  if (d->dtype != LLAMA_BF16) return LLAMA_ERR_UNSUPPORTED;
  // every input dimension is cut into whole groups of 64
  if (d->dim % 64 || d->ffn_dim % 64 || (d->n_heads * d->head_dim) % 64) return LLAMA_ERR_UNSUPPORTED;
  return LLAMA_OK;
}

// Decode step of one block whose seven projections hold 4-bit group-64
// weights: the same sequence as run_layer's bf16 decode path, each
// projection on gemm_q4_kernel.
llama_status run_layer_decode_q4(const llama_dims& d, const llama_layer_weights_q4& w, llama_kv_cache* kv, int B,
                                 const float* x_in, float* x_out, uint8_t* ws, const WsLayout& lay,
                                 cudaStream_t st) {
  using bf = __nv_bfloat16;
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  const int nh = d.n_heads, nkv = d.n_kv_heads, hd = d.head_dim;
  const int qkvn = (nh + 2 * nkv) * hd;
  const int p0 = kv->length;
  bf* qkv = reinterpret_cast<bf*>(ws + lay.qkv);
  bf* h = reinterpret_cast<bf*>(ws + lay.h);
  bf* att = reinterpret_cast<bf*>(ws + lay.attn);
  bf* mb = reinterpret_cast<bf*>(ws + lay.mbuf);
  const SkScratch part{reinterpret_cast<float*>(ws + lay.partial), reinterpret_cast<unsigned*>(ws + lay.sk_flags),
                         reinterpret_cast<float*>(ws + lay.ssq)};
  {
    TRACE(K_RMSNORM, st);
    CUDA_TRY(launch_k(rmsnorm_kernel<bf>, B, rmsnorm_threads(d.dim), 0, st, x_in, d.dim, w.attn_norm, h, B, d.dim,
                      d.eps, RopeTab{nullptr, 0, 0, 0, 0.f, early_trigger()}));
  }
  LAUNCH_CHECK();
  const Q4Seg sq[3] = {{w.wq, nh * hd, 0}, {w.wk, nkv * hd, nh * hd}, {w.wv, nkv * hd, (nh + nkv) * hd}};
  TRY(gemm_decode_q4(st, h, B, d.dim, sq, 3, EPI_BF16, qkv, qkvn, nullptr, 0, part, status, K_GEMM_QKV));
  const bool rope_in_attn = decode_rope_fusable(d, B, p0 + 1);
  const RopeFuse rf{d.rope_theta, d.rope_style};
  if (!rope_in_attn) {
    TRACE(K_ROPE_APPEND, st);
    CUDA_TRY(launch_k(rope_append_kernel<bf>, B, 256, 0, st, qkv, reinterpret_cast<bf*>(kv->k),
                      reinterpret_cast<bf*>(kv->v), 1, p0, nh, nkv, hd, kv->capacity, d.rope_theta, d.rope_style,
                      static_cast<const SeqTab*>(nullptr)));
    LAUNCH_CHECK();
  }
  TRY(attn_decode_bf16(st, d, kv->k, kv->v, kv->capacity, B, p0 + 1, qkv, qkvn, att,
                       reinterpret_cast<float*>(ws + lay.att_ml), reinterpret_cast<float*>(ws + lay.att_o), status,
                       1, kMaxAttnSplits, nullptr, rope_in_attn ? &rf : nullptr));
  // o_proj + residual, with RMSNorm-2 at its end
  const Q4Seg so{w.wo, d.dim, 0};
  const bool fuse_norm = norm_fusable(d, B);
  const NormFuse n2{w.ffn_norm, h, d.eps};
  TRY(gemm_decode_q4(st, att, B, nh * hd, &so, 1, EPI_RESID_F32, x_out, d.dim, x_in, d.dim, part, status, K_GEMM_O,
                     fuse_norm ? &n2 : nullptr));
  if (!fuse_norm) {
    TRACE(K_RMSNORM, st);
    CUDA_TRY(launch_k(rmsnorm_kernel<bf>, B, rmsnorm_threads(d.dim), 0, st, x_out, d.dim, w.ffn_norm, h, B, d.dim,
                      d.eps, RopeTab{nullptr, 0, 0, 0, 0.f, early_trigger()}));
    LAUNCH_CHECK();
  }
  const Q4Seg sg[2] = {{w.w1, d.ffn_dim, 0}, {w.w3, d.ffn_dim, 0}};
  TRY(gemm_decode_q4(st, h, B, d.dim, sg, 2, EPI_SWIGLU_BF16, mb, d.ffn_dim, nullptr, 0, part, status,
                     K_GEMM_GATE_UP));
  const Q4Seg sd{w.w2, d.dim, 0};
  TRY(gemm_decode_q4(st, mb, B, d.ffn_dim, &sd, 1, EPI_RESID_F32, x_out, d.dim, x_out, d.dim, part, status,
                     K_GEMM_DOWN));
  kv->length = p0 + 1;
  return LLAMA_OK;
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

int32_t llama_abi_version(void) { return LLAMA_B200_ABI_VERSION; }

const char* llama_status_string(llama_status s) {
  switch (s) {
    case LLAMA_OK: return "ok";
    case LLAMA_ERR_INVALID_ARG: return "invalid argument";
    case LLAMA_ERR_UNSUPPORTED: return "unsupported configuration";
    case LLAMA_ERR_CACHE_FULL: return "KV cache full";
    case LLAMA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case LLAMA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case LLAMA_ERR_CUDA: return "CUDA error";
    case LLAMA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case LLAMA_ERR_SCRATCH_LIMIT: return "request exceeds the fixed scratch of the allocation-free entry point";
  }
  return "unknown status";
}

uint64_t llama_set_wait_limit_ns(uint64_t ns) { return g_wait_limit_ns.exchange(ns == 0 ? 1 : ns); }

uint64_t llama_launch_count(void) { return g_launch_count.load(); }

llama_status llama_profile_enable(int32_t on) {
  Tracer& t = tracer();
  std::lock_guard<std::mutex> g(t.mu);
  t.on = on != 0;
  return LLAMA_OK;
}

int32_t llama_profile_inflight(const char** names, int32_t n) {
  Tracer& t = tracer();
  std::lock_guard<std::mutex> g(t.mu);
  int32_t k = 0;
  for (const ProfRec& r : t.pending) {
    const cudaError_t e = cudaEventQuery(r.b);
    if (e == cudaErrorNotReady) {
      if (names && k < n) names[k] = kKindNames[r.kind];
      ++k;
    } else if (e != cudaSuccess) {
      (void)cudaGetLastError();
    }
  }
  return k;
}

int32_t llama_profile_read(const char** names, double* total_ms, long long* launches, int32_t n, int32_t reset) {
  Tracer& t = tracer();
  std::lock_guard<std::mutex> g(t.mu);
  for (ProfRec& r : t.pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      t.total_ms[r.kind] += ms;
      t.launches[r.kind] += 1;
    } else {
      (void)cudaGetLastError();
    }
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  t.pending.clear();
  for (int i = 0; i < n && i < K_COUNT; ++i) {
    if (names) names[i] = kKindNames[i];
    if (total_ms) total_ms[i] = t.total_ms[i];
    if (launches) launches[i] = t.launches[i];
  }
  if (reset) {
    for (int i = 0; i < K_COUNT; ++i) {
      t.total_ms[i] = 0.0;
      t.launches[i] = 0;
    }
  }
  return K_COUNT;
}

llama_status llama_kv_cache_create(const llama_dims* dims, int32_t batch, int32_t capacity, void* k_buf,
                                   void* v_buf, llama_kv_cache** out) {
  if (out == nullptr) return LLAMA_ERR_INVALID_ARG;
  *out = nullptr;
  TRY(check_dims(dims));
  if (batch <= 0 || capacity <= 0 || k_buf == nullptr || v_buf == nullptr) return LLAMA_ERR_INVALID_ARG;
  if (!aligned16(k_buf) || !aligned16(v_buf)) return LLAMA_ERR_ALIGNMENT;
  auto* c = new (std::nothrow) llama_kv_cache;
  if (c == nullptr) return LLAMA_ERR_INVALID_ARG;
  c->dims = *dims;
  c->batch = batch;
  c->capacity = capacity;
  c->length = 0;
  c->k = k_buf;
  c->v = v_buf;
  *out = c;
  return LLAMA_OK;
}

llama_status llama_kv_cache_set_length(llama_kv_cache* c, int32_t len) {
  if (c == nullptr || len < 0) return LLAMA_ERR_INVALID_ARG;
  if (len > c->capacity) return LLAMA_ERR_CACHE_FULL;
  c->length = len;
  c->lens.clear();
  return LLAMA_OK;
}

llama_status llama_kv_cache_set_lengths(llama_kv_cache* c, const int32_t* lens) {
  if (c == nullptr || lens == nullptr) return LLAMA_ERR_INVALID_ARG;
  bool same = true;
  for (int b = 0; b < c->batch; ++b) {
    if (lens[b] < 0) return LLAMA_ERR_INVALID_ARG;
    if (lens[b] > c->capacity) return LLAMA_ERR_CACHE_FULL;
    same = same && lens[b] == lens[0];
  }
  if (same) {
    c->length = lens[0];
    c->lens.clear();
  } else {
    c->length = -2;
    c->lens.assign(lens, lens + c->batch);
  }
  return LLAMA_OK;
}

llama_status llama_kv_cache_lengths(const llama_kv_cache* c, int32_t* lens) {
  if (c == nullptr || lens == nullptr) return LLAMA_ERR_INVALID_ARG;
  for (int b = 0; b < c->batch; ++b) lens[b] = c->lens.empty() ? c->length : c->lens[b];
  return LLAMA_OK;
}

int32_t llama_kv_cache_length(const llama_kv_cache* c) { return c ? c->length : -1; }
int32_t llama_kv_cache_capacity(const llama_kv_cache* c) { return c ? c->capacity : -1; }
void llama_kv_cache_destroy(llama_kv_cache* c) { delete c; }

size_t llama_workspace_size(const llama_dims* dims, int32_t batch, int32_t seq_len) {
  if (check_dims(dims) != LLAMA_OK || batch <= 0 || seq_len <= 0) return 0;
  return plan_ws(*dims, batch, seq_len, 0).total;
}

llama_status llama_workspace_offsets(const llama_dims* dims, int32_t batch, int32_t seq_len, size_t* out,
                                     int32_t n) {
  TRY(check_dims(dims));
  if (batch <= 0 || seq_len <= 0 || out == nullptr || n < 0) return LLAMA_ERR_INVALID_ARG;
  const WsLayout w = plan_ws(*dims, batch, seq_len, 0);
  const size_t v[4] = {w.qkv, w.h, w.attn, w.mbuf};
  for (int i = 0; i < n && i < 4; ++i) out[i] = v[i];
  return LLAMA_OK;
}

llama_status llama_device_status(const void* workspace, int32_t clear) {
  if (workspace == nullptr) return LLAMA_ERR_INVALID_ARG;
  DevStatus s{};
  CUDA_TRY(cudaMemcpy(&s, workspace, sizeof(s), cudaMemcpyDeviceToHost));
  if (clear) {
    DevStatus z{};
    CUDA_TRY(cudaMemcpy(const_cast<void*>(workspace), &z, sizeof(z), cudaMemcpyHostToDevice));
  }
  return static_cast<llama_status>(s.code);
}

llama_status llama_layer_prefill(const llama_dims* dims, const llama_layer_weights* w, llama_kv_cache* cache,
                                 int32_t batch, int32_t seq_len, const float* x_in, float* x_out, void* workspace,
                                 size_t ws_bytes, void* stream) {
  TRY(check_layer_call(dims, w, cache, batch, seq_len, x_in, x_out, workspace, ws_bytes, 0));
  const WsLayout lay = plan_ws(*dims, batch, seq_len, 0);
  return run_layer(*dims, *w, cache, batch, seq_len, x_in, x_out, static_cast<uint8_t*>(workspace), lay,
                   static_cast<cudaStream_t>(stream));
}

llama_status llama_layer_decode(const llama_dims* dims, const llama_layer_weights* w, llama_kv_cache* cache,
                                int32_t batch, const float* x_in, float* x_out, void* workspace, size_t ws_bytes,
                                void* stream) {
  TRY(check_layer_call(dims, w, cache, batch, 1, x_in, x_out, workspace, ws_bytes, 0));
  const WsLayout lay = plan_ws(*dims, batch, 1, 0);
  return run_layer(*dims, *w, cache, batch, 1, x_in, x_out, static_cast<uint8_t*>(workspace), lay,
                   static_cast<cudaStream_t>(stream));
}

llama_status llama_layer_decode_q4(const llama_dims* dims, const llama_layer_weights_q4* w, llama_kv_cache* cache,
                                   int32_t batch, const float* x_in, float* x_out, void* workspace, size_t ws_bytes,
                                   void* stream) {
  TRY(check_layer_q4(dims, w));
  if (cache == nullptr || x_in == nullptr || x_out == nullptr || workspace == nullptr || batch <= 0)
    return LLAMA_ERR_INVALID_ARG;
  if (batch > kSwapMaxTokens) return LLAMA_ERR_UNSUPPORTED;
  if (!same_dims(*dims, cache->dims) || batch != cache->batch || !cache->lens.empty()) return LLAMA_ERR_INVALID_ARG;
  if (!aligned16(x_in) || !aligned16(x_out) || !aligned16(workspace)) return LLAMA_ERR_ALIGNMENT;
  const size_t xb = (size_t)batch * dims->dim * 4;
  if (overlap(x_in, xb, x_out, xb)) return LLAMA_ERR_INVALID_ARG;
  if ((long long)cache->length + 1 > cache->capacity) return LLAMA_ERR_CACHE_FULL;
  const WsLayout lay = plan_ws(*dims, batch, 1, 0);
  if (ws_bytes < lay.total) return LLAMA_ERR_WORKSPACE_TOO_SMALL;
  return run_layer_decode_q4(*dims, *w, cache, batch, x_in, x_out, static_cast<uint8_t*>(workspace), lay,
                             static_cast<cudaStream_t>(stream));
}

size_t llama_workspace_size_ragged(const llama_dims* dims, int32_t batch, int32_t total_tokens) {
  if (check_dims(dims) != LLAMA_OK || batch <= 0 || batch > kMaxRagged || total_tokens < batch) return 0;
  return plan_ws(*dims, batch, 1, 0, total_tokens).total;
}

llama_status llama_layer_forward_ragged(const llama_dims* dims, const llama_layer_weights* w, llama_kv_cache* cache,
                                        int32_t batch, const int32_t* n_new, const float* x_in, float* x_out,
                                        void* workspace, size_t ws_bytes, void* stream) {
  TRY(check_dims(dims));
  TRY(check_weights(w));
  if (cache == nullptr || n_new == nullptr || x_in == nullptr || x_out == nullptr || workspace == nullptr)
    return LLAMA_ERR_INVALID_ARG;
  if (dims->dtype != LLAMA_BF16) return LLAMA_ERR_UNSUPPORTED;
  if (batch <= 0 || batch != cache->batch || !same_dims(*dims, cache->dims)) return LLAMA_ERR_INVALID_ARG;
  if (batch > kMaxRagged) return LLAMA_ERR_UNSUPPORTED;
  long long M = 0;
  for (int b = 0; b < batch; ++b) {
    if (n_new[b] < 1) return LLAMA_ERR_INVALID_ARG;
    const long long p0 = cache->lens.empty() ? cache->length : cache->lens[b];
    if (p0 + n_new[b] > cache->capacity) return LLAMA_ERR_CACHE_FULL;
    M += n_new[b];
  }
  if (M > (1LL << 30)) return LLAMA_ERR_UNSUPPORTED;
  if (!aligned16(x_in) || !aligned16(x_out) || !aligned16(workspace)) return LLAMA_ERR_ALIGNMENT;
  const size_t xb = (size_t)M * dims->dim * 4;
  if (overlap(x_in, xb, x_out, xb)) return LLAMA_ERR_INVALID_ARG;
  const WsLayout lay = plan_ws(*dims, batch, 1, 0, (int)M);
  if (ws_bytes < lay.total) return LLAMA_ERR_WORKSPACE_TOO_SMALL;
  return run_layer_ragged(*dims, *w, cache, batch, n_new, x_in, x_out, static_cast<uint8_t*>(workspace), lay,
                          static_cast<cudaStream_t>(stream));
}

size_t llama_model_workspace_size(const llama_model* m, int32_t batch, int32_t seq_len) {
  if (m == nullptr || check_dims(&m->dims) != LLAMA_OK || batch <= 0 || seq_len <= 0 || m->vocab <= 0) return 0;
  return plan_ws(m->dims, batch, seq_len, m->vocab).total;
}

}  // extern "C"

namespace {

// Next-token choice after the lm_head: greedy argmax, or temperature / top-p
// sampling with one uniform per sequence.
struct TokenPick {
  float temperature;   // 0: argmax
  float top_p;
  const float* u;      // device [batch]
};

llama_status check_pick(const TokenPick& pk, int batch) {
  if (!(pk.temperature >= 0.f) || !(pk.temperature < 1e30f)) return LLAMA_ERR_INVALID_ARG;
  if (pk.temperature > 0.f) {
    if (!(pk.top_p > 0.f) || !(pk.top_p <= 1.f) || pk.u == nullptr) return LLAMA_ERR_INVALID_ARG;
    if (!aligned16(pk.u)) return LLAMA_ERR_ALIGNMENT;
  }
  (void)batch;
  return LLAMA_OK;
}

llama_status enqueue_pick(const TokenPick& pk, const float* logits, int batch, int vocab, int32_t* ids,
                          cudaStream_t st) {
  if (pk.temperature == 0.f) {
    TRACE(K_ARGMAX, st);
    CUDA_TRY(launch_k(argmax_kernel, batch, 1024, 0, st, logits, vocab, ids));
  } else {
    TRACE(K_SAMPLE, st);
    CUDA_TRY(launch_k(sample_top_p_kernel, batch, SAMPLE_THREADS, 0, st, logits, vocab, pk.temperature, pk.top_p,
                      pk.u, ids));
  }
  LAUNCH_CHECK();
  return LLAMA_OK;
}

llama_status model_forward(const llama_model* m, llama_kv_cache* const* caches, const int32_t* tokens,
                           int32_t batch, int32_t seq_len, float* logits_or_null, int32_t* next_ids,
                           void* workspace, size_t ws_bytes, void* stream, const TokenPick& pick) {
  if (m == nullptr || caches == nullptr || tokens == nullptr || next_ids == nullptr || workspace == nullptr)
    return LLAMA_ERR_INVALID_ARG;
  TRY(check_dims(&m->dims));
  const llama_dims& d = m->dims;
  if (m->n_layers <= 0 || m->vocab <= 0 || m->layers == nullptr || m->embed == nullptr ||
      m->final_norm == nullptr || m->lm_head == nullptr)
    return LLAMA_ERR_INVALID_ARG;
  if (batch <= 0 || seq_len <= 0) return LLAMA_ERR_INVALID_ARG;
  if (!aligned16(m->embed) || !aligned16(m->final_norm) || !aligned16(m->lm_head) || !aligned16(tokens) ||
      !aligned16(next_ids) || !aligned16(workspace) || (logits_or_null && !aligned16(logits_or_null)))
    return LLAMA_ERR_ALIGNMENT;
  const WsLayout lay = plan_ws(d, batch, seq_len, m->vocab);
  if (ws_bytes < lay.total) return LLAMA_ERR_WORKSPACE_TOO_SMALL;
  const int len0 = caches[0] ? caches[0]->length : -1;
  for (int l = 0; l < m->n_layers; ++l) {
    llama_kv_cache* c = caches[l];
    if (c == nullptr || !same_dims(c->dims, d) || c->batch != batch || c->length != len0 || !c->lens.empty())
      return LLAMA_ERR_INVALID_ARG;
    if ((long long)c->length + seq_len > c->capacity) return LLAMA_ERR_CACHE_FULL;
    TRY(check_weights(&m->layers[l]));
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  const int M = batch * seq_len;
  float* xa = reinterpret_cast<float*>(ws + lay.xa);
  float* xb = reinterpret_cast<float*>(ws + lay.xb);
  // a1: embedding
  {
  TRACE(K_EMBED, st);
  if (d.dtype == LLAMA_BF16)
    CUDA_TRY(launch_k(embed_kernel<__nv_bfloat16>, cdiv(M, 8), 256, 0, st, 
        tokens, static_cast<const __nv_bfloat16*>(m->embed), xa, M, d.dim, m->vocab, status));
  else
    embed_kernel<float><<<cdiv(M, 8), 256, 0, st>>>(tokens, static_cast<const float*>(m->embed), xa, M, d.dim,
                                                    m->vocab, status);
  }
  LAUNCH_CHECK();
  // blocks (decode with fused norms: each block's down GEMM ends with the next
  // block's RMSNorm-1, the last one with the final RMSNorm into the lm_head's input)
  const bool chain = d.dtype == LLAMA_BF16 && seq_len == 1 && norm_fusable(d, batch);
  void* hbuf = ws + lay.h;
  void* hl_buf = ws + lay.hl;
  for (int l = 0; l < m->n_layers; ++l) {
    const bool last = l + 1 == m->n_layers;
    const float* nn = chain ? (last ? m->final_norm : m->layers[l + 1].attn_norm) : nullptr;
    // without the chained norms: each down GEMM leaves its rows' sums of
    // squares for the next block's QKV GEMM, which then does RMSNorm-1 itself
    TRY(run_layer(d, m->layers[l], caches[l], batch, seq_len, xa, xb, ws, lay, st, nn, last ? hl_buf : hbuf,
                  chain && l > 0, !chain && l > 0, !chain && !last));
    std::swap(xa, xb);
  }
  // a10: final norm + lm_head on the last row of each sequence + argmax
  const float* xl = xa;
  if (seq_len > 1) {
    float* g = reinterpret_cast<float*>(ws + lay.xl);
    {
      TRACE(K_GATHER_LAST, st);
      CUDA_TRY(launch_k(gather_last_rows_kernel, dim3(cdiv(d.dim, 256), batch), 256, 0, st, xa, g, seq_len, d.dim));
    }
    LAUNCH_CHECK();
    xl = g;
  }
  float* logits = logits_or_null ? logits_or_null : reinterpret_cast<float*>(ws + lay.logits);
  if (d.dtype == LLAMA_BF16) {
    __nv_bfloat16* hl = reinterpret_cast<__nv_bfloat16*>(ws + lay.hl);
    if (!chain) {
      TRACE(K_RMSNORM, st);
      CUDA_TRY(launch_k(rmsnorm_kernel<__nv_bfloat16>, batch, rmsnorm_threads(d.dim), 0, st, xl, d.dim,
                        m->final_norm, hl, batch, d.dim, d.eps, RopeTab{nullptr, 0, 0, 0, 0.f, early_trigger()}));
      LAUNCH_CHECK();
    }
    WSeg s{m->lm_head, m->vocab, 0};
    TRY(gemm_bf16(st, true, hl, batch, d.dim, &s, 1, EPI_F32, logits, m->vocab, nullptr, 0,
                  SkScratch{reinterpret_cast<float*>(ws + lay.partial), reinterpret_cast<unsigned*>(ws + lay.sk_flags)},
                  status, K_GEMM_LM_HEAD));
  } else {
    float* hl = reinterpret_cast<float*>(ws + lay.hl);
    {
      TRACE(K_RMSNORM, st);
      rmsnorm_kernel<float><<<batch, rmsnorm_threads(d.dim), 0, st>>>(xl, d.dim, m->final_norm, hl, batch, d.dim,
                                                                      d.eps, RopeTab{});
    }
    {
      TRACE(K_GEMM_LM_HEAD, st);
      gemm_f32_kernel<F32_STORE><<<dim3(cdiv(m->vocab, 64), cdiv(batch, 64)), 256, 0, st>>>(
          hl, d.dim, static_cast<const float*>(m->lm_head), nullptr, d.dim, batch, m->vocab, d.dim, logits,
          m->vocab, nullptr, 0);
    }
    LAUNCH_CHECK();
  }
  return enqueue_pick(pick, logits, batch, m->vocab, next_ids, st);
}

}  // namespace

extern "C" {

llama_status llama_model_forward(const llama_model* m, llama_kv_cache* const* caches, const int32_t* tokens,
                                 int32_t batch, int32_t seq_len, float* logits_or_null, int32_t* next_ids,
                                 void* workspace, size_t ws_bytes, void* stream) {
  return model_forward(m, caches, tokens, batch, seq_len, logits_or_null, next_ids, workspace, ws_bytes, stream,
                       TokenPick{0.f, 1.f, nullptr});
}

llama_status llama_model_forward_sample(const llama_model* m, llama_kv_cache* const* caches, const int32_t* tokens,
                                        int32_t batch, int32_t seq_len, float temperature, float top_p,
                                        const float* u, float* logits_or_null, int32_t* next_ids, void* workspace,
                                        size_t ws_bytes, void* stream) {
  const TokenPick pk{temperature, top_p, u};
  TRY(check_pick(pk, batch));
  return model_forward(m, caches, tokens, batch, seq_len, logits_or_null, next_ids, workspace, ws_bytes, stream,
                       pk);
}

llama_status llama_sample_top_p(const float* logits, int32_t batch, int32_t vocab, float temperature, float top_p,
                                const float* u, int32_t* ids, void* stream) {
  if (logits == nullptr || ids == nullptr || batch <= 0 || vocab <= 0) return LLAMA_ERR_INVALID_ARG;
  if (!aligned16(logits) || !aligned16(ids)) return LLAMA_ERR_ALIGNMENT;
  const TokenPick pk{temperature, top_p, u};
  TRY(check_pick(pk, batch));
  return enqueue_pick(pk, logits, batch, vocab, ids, static_cast<cudaStream_t>(stream));
}

llama_status llama_selftest_wait_timeout(void* workspace, uint64_t limit_ns, void* stream) {
  if (workspace == nullptr) return LLAMA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return LLAMA_ERR_ALIGNMENT;
  if (limit_ns > 5000000000ull) return LLAMA_ERR_INVALID_ARG;
  {
    TRACE(K_SELFTEST, static_cast<cudaStream_t>(stream));
    selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(reinterpret_cast<DevStatus*>(workspace),
                                                                        limit_ns);
  }
  LAUNCH_CHECK();
  return LLAMA_OK;
}

}  // extern "C"

// ====================================================================== decode attention, no allocation
//
// For callers that cannot allocate device memory at all -- for example code
// running inside a serving framework that has reserved all GPU memory for its
// own pool and gives a plug-in no workspace, or a real-time loop that must not
// call cudaMalloc (which can synchronise the device) -- this variant of the
// split-KV decode attention keeps its partial results in a fixed array that is
// part of the library image instead of in a caller-provided workspace.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB, held on every GPU that loads the library
__device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
llama_status noalloc_scratch(float** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices) return LLAMA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return LLAMA_OK;
}

}  // namespace

extern "C" llama_status llama_attention_decode_noalloc(const llama_dims* dims, int32_t batch, const void* q,
                                                       int32_t ld_q, const void* k_cache, const void* v_cache,
                                                       int32_t capacity, int32_t length, void* out, void* stream) {
  TRY(check_dims(dims));
  const llama_dims& d = *dims;
  if (d.dtype != LLAMA_BF16) return LLAMA_ERR_UNSUPPORTED;
  if (batch <= 0 || q == nullptr || k_cache == nullptr || v_cache == nullptr || out == nullptr)
    return LLAMA_ERR_INVALID_ARG;
  if (length <= 0 || capacity < length || ld_q < d.n_heads * d.head_dim) return LLAMA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || (ld_q % 8) != 0)
    return LLAMA_ERR_ALIGNMENT;
  const int hd = d.head_dim;
  // partials of `splits` key ranges per (sequence, query head): (max, sum) and hd outputs
  const size_t per_split = (size_t)batch * d.n_heads * (hd + 2) * sizeof(float);
  const size_t max_splits = kNoAllocScratchBytes / per_split;
  if (max_splits < 2) return LLAMA_ERR_SCRATCH_LIMIT;
  const int cap_splits = (int)std::min<size_t>(max_splits, kMaxAttnSplits);
  float* scratch = nullptr;
  TRY(noalloc_scratch(&scratch));
  float* part_ml = scratch;
  float* part_o = scratch + (size_t)batch * d.n_heads * cap_splits * 2;
  // the same kernels and split heuristic as llama_layer_decode, with at least two splits (the
  // partials live in the fixed array); no workspace, so no device status word is written
  return attn_decode_bf16(static_cast<cudaStream_t>(stream), d, k_cache, v_cache, capacity, batch, length,
                          static_cast<const __nv_bfloat16*>(q), ld_q, static_cast<__nv_bfloat16*>(out), part_ml,
                          part_o, nullptr, 2, cap_splits);
}
