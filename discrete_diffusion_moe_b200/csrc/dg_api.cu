// dg_api.cu - host side of the library: weight / workspace layouts, TMA
// tensor maps, kernel orchestration of one denoising round, context encoding
// and the block loop, behind the C ABI of include/dg.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <set>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/dg.h"
#include "../../include/dg_testing.h"
#include "../../synth/synth.h"
#include "attention_tc.cuh"
#include "epilogues.cuh"
#include "gemm_pair.cuh"
#include "gemm_tc.cuh"
#include "moe_pair.cuh"
#include "kernels.cuh"

using namespace dg;

// ============================================================================
// errors
static thread_local char g_err[512] = "";

static dg_status fail(dg_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

#define DG_CUDA(call)                                                                        \
  do {                                                                                       \
    cudaError_t e_ = (call);                                                                 \
    if (e_ != cudaSuccess) return fail(DG_ERR_CUDA, "%s: %s (%s:%d)", #call,                \
                                       cudaGetErrorString(e_), __FILE__, __LINE__);          \
  } while (0)

#define DG_TRY(expr)                  \
  do {                                \
    dg_status s_ = (expr);            \
    if (s_ != DG_OK) return s_;       \
  } while (0)

extern "C" const char* dg_last_error(void) { return g_err; }

// NVTX range over one phase of the method (host side: brackets the phase's
// launches for a profiler's timeline; a no-op when no tool is attached)
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// One kernel launch.  With DG_PDL (programmatic dependent launch) its CTAs
// may be scheduled while the stream's previous kernel finishes: every kernel
// of the library waits (griddepcontrol.wait) before it touches memory that
// another kernel writes, so only its launch latency and its own set-up
// (barriers, tensor memory, tensor-map prefetch) overlap the predecessor's
// tail.  Optional cluster shape and cluster scheduling policy.
#ifndef DG_PDL
#define DG_PDL 1
#endif
// 1: the QKV and output projections run on CTA pairs (each CTA of a pair
// copies half of the unit's token rows), with the same k splits and partials
#ifndef DG_PROJ_PAIR
#define DG_PROJ_PAIR 0
#endif
// most k splits of the output projection (its partials are summed by the
// residual + RMSNorm kernel, which takes any count)
#ifndef DG_O_SPLITS
#define DG_O_SPLITS 3
#endif
// 1: the two grouped expert products run as one persistent launch on CTA
// pairs (moe_pair.cuh), a chunk's down product starting as soon as its
// gate/up outputs are stored
#ifndef DG_MOE_FUSED
#define DG_MOE_FUSED 1
#endif
// token rows per grouped (expert) unit: 0 chooses 128 on CTA pairs, or 256 on
// single CTAs when experts average more than 64 tokens; 256 takes 256-token
// chunks on CTA pairs (one read of an expert's weight tile for up to 256 tokens)
#ifndef DG_GROUPED_BN
#define DG_GROUPED_BN 0
#endif
struct Launch {
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute at[3];
  Launch(dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl = DG_PDL) {
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    lc.attrs = at;
    if (pdl) {
      at[lc.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      at[lc.numAttrs].val.programmaticStreamSerializationAllowed = 1;
      ++lc.numAttrs;
    }
  }
  Launch& cluster(unsigned x, unsigned y, unsigned z) {
    at[lc.numAttrs].id = cudaLaunchAttributeClusterDimension;
    at[lc.numAttrs].val.clusterDim.x = x;
    at[lc.numAttrs].val.clusterDim.y = y;
    at[lc.numAttrs].val.clusterDim.z = z;
    ++lc.numAttrs;
    return *this;
  }
  Launch& policy(cudaClusterSchedulingPolicy pol) {
    at[lc.numAttrs].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    at[lc.numAttrs].val.clusterSchedulingPolicyPreference = pol;
    ++lc.numAttrs;
    return *this;
  }
  template <typename... KArgs, typename... Args>
  cudaError_t operator()(void (*k)(KArgs...), Args&&... args) {
    return cudaLaunchKernelEx(&lc, k, std::forward<Args>(args)...);
  }
};

// ============================================================================
// configuration checks and layouts
static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
static int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

static bool cfg_ok(const dg_model_config* c, char* why, size_t n) {
  if (!c) { snprintf(why, n, "null config"); return false; }
  if (c->n_layers < 1 || c->d_model < 256 || c->d_model % 64 || c->d_model > 4096) { snprintf(why, n, "d_model must be a multiple of 64 in [256, 4096]"); return false; }
  if (c->head_dim < 16 || c->head_dim % 16 || c->head_dim > 256) { snprintf(why, n, "head_dim must be a multiple of 16 in [16, 256]"); return false; }
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 176) {
    snprintf(why, n, "head_dim %d not built (32, 64, 128, 176)", c->head_dim); return false;
  }
  if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads) { snprintf(why, n, "n_q_heads must be a multiple of n_kv_heads"); return false; }
  if ((c->n_q_heads * c->head_dim) % 64) { snprintf(why, n, "n_q_heads * head_dim must be a multiple of 64"); return false; }
  if (c->n_experts < 1 || c->n_experts > 256) { snprintf(why, n, "n_experts must be in [1, 256]"); return false; }
  if (c->top_k < 1 || c->top_k > 8 || c->top_k > c->n_experts) { snprintf(why, n, "top_k must be in [1, min(8, n_experts)]"); return false; }
  if (c->d_ff < 64 || c->d_ff % 64) { snprintf(why, n, "d_ff must be a multiple of 64"); return false; }
  if (c->vocab < 256 || c->vocab % 256) { snprintf(why, n, "vocab must be a multiple of 256"); return false; }
  if (!(c->rope_theta > 0.f) || !(c->rms_eps > 0.f)) { snprintf(why, n, "rope_theta and rms_eps must be > 0"); return false; }
  return true;
}

namespace {

struct LayerW {
  size_t wqkv, wo, wr, wgu, wd, g_attn, g_moe;
};
struct WLayout {
  size_t emb, embT, lm, sc, g_final;
  std::vector<LayerW> layers;
  size_t total;  // elements
  int qkv_rows, wr_rows;
};

WLayout weight_layout(const dg_model_config& c) {
  WLayout w;
  size_t off = 0;
  auto take = [&](size_t n) { size_t o = off; off = align_up(off + n, 128); return o; };
  const size_t d = c.d_model, V = c.vocab;
  w.qkv_rows = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim;
  w.wr_rows = (int)align_up(c.n_experts, 128);
  w.emb = take(V * d);
  w.embT = take(V * d);
  w.lm = take(V * d);
  w.sc = c.self_cond ? take(d * d) : 0;
  w.g_final = take(d);
  for (int l = 0; l < c.n_layers; ++l) {
    LayerW L;
    L.wqkv = take((size_t)w.qkv_rows * d);
    L.wo = take(d * (size_t)c.n_q_heads * c.head_dim);
    L.wr = take((size_t)w.wr_rows * d);
    L.wgu = take((size_t)c.n_experts * 2 * c.d_ff * d);
    L.wd = take((size_t)c.n_experts * d * c.d_ff);
    L.g_attn = take(d);
    L.g_moe = take(d);
    w.layers.push_back(L);
  }
  w.total = off;
  return w;
}

constexpr int kMaxAttnSplits = 8;

struct WsLayout {
  size_t err, flags, x, xn, qkv, opart, q, attn, rpart, tok, xnc, rbar, rfill, off, choff, perm, inv, wperm,
      xperm, hperm, yperm, logits, vp_m, vp_z, vp_s, vp_av, vp_ai, vp_gv, vp_gi, st_m, st_iz, st_h,
      st_pmax, st_amax, st_samp, probs, epart, rope, stepdev, dstat, dep, total;
  int T_alloc, P_alloc, ks_r, n_vt;  // T_alloc: token rows of a layer pass (>= the canvas tokens)
  int T_canvas;                       // canvas tokens (batch * 256): rows of the vocabulary buffers
  long long epart_rows;
};

// split-k of the router product: 8 from 16 k-blocks on (d_model >= 1024), else 4
// (d_model >= 256); the routing kernel is built for both
int router_splits(const dg_model_config& c) { return std::min(c.d_model >= 1024 ? 8 : 4, c.d_model / 64); }

// Cluster scheduling preference of the split-k projections (1: pack the
// CTAs of clusters onto SMs to balance load, 0: spread them over SMs).
#ifndef DG_CLUSTER_POLICY
#define DG_CLUSTER_POLICY 1
#endif
// How the split-k projections are summed: 1 = the k splits of a tile form a
// thread-block cluster and add their accumulators through distributed shared
// memory (the QKV projection then applies RoPE and writes q / K / V^T in its
// epilogue); 0 = each split writes fp32 partials that the next kernel sums
// (RoPE / KV write, residual + RMSNorm, routing).
#ifndef DG_QKV_CLUSTER
#define DG_QKV_CLUSTER 0
#endif
#ifndef DG_O_CLUSTER
#define DG_O_CLUSTER 0
#endif
#ifndef DG_ROUTER_CLUSTER
#define DG_ROUTER_CLUSTER 0
#endif
// Largest token tile of the QKV and output projections.
#ifndef DG_PROJ_BN_MAX
#define DG_PROJ_BN_MAX 128
#endif

// Token columns per unit of the QKV and output projections: 128 from 256
// tokens on (two CTAs share an SM, each weight tile is read by two CTAs at the
// same time, the second time from L2).
int proj_bn(int T) { return T >= 256 ? DG_PROJ_BN_MAX : std::min(256, std::max(16, next_pow2(T))); }

// Split-k of the QKV and output projections: enough units for two CTAs per
// SM, at most 3 (every split is one more fp32 partial its consumer reads).
int proj_splits(int m_tiles, int T, int kb, int num_sms, int cap = 3) {
  const int n_tiles = (T + proj_bn(T) - 1) / proj_bn(T);
  const int ks = (2 * num_sms) / std::max(1, m_tiles * n_tiles);
  return std::max(1, std::min({ks, cap, kb / 4}));
}

// Split-k (over the vocabulary) of the expected-embedding product
// e = probs . E_emb: units of two 128-row tiles of E_emb^T (one token tile
// feeding both) and about one unit per SM (one CTA per SM: the two
// accumulators of 256 columns fill the tensor memory).
constexpr int kEsumMt = 2;
int esum_splits(const dg_model_config& c, int T, int num_sms) {
  const int m_units = ((c.d_model + 127) / 128 + kEsumMt - 1) / kEsumMt;
  const int bn = std::min(256, std::max(16, next_pow2(T)));
  const int n_tiles = (T + bn - 1) / bn;
  int ks = num_sms / std::max(1, m_units * n_tiles);
  ks = std::max(1, std::min(ks, 32));
  return std::min(ks, c.vocab / 64);
}

// Workspace of a context for up to `batch` canvases whose causal encode passes
// take up to `prefill` tokens (all canvases together; at least batch * 256).
WsLayout ws_layout(const dg_model_config& c, int batch, int num_sms, int prefill = 0) {
  WsLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  const size_t Tc = (size_t)batch * DG_CANVAS;                          // canvas tokens
  const size_t T = std::max(Tc, (size_t)align_up((size_t)std::max(prefill, 0), DG_CANVAS));  // layer rows
  const size_t d = c.d_model, V = c.vocab, k = c.top_k, E = c.n_experts;
  const size_t P = T * k;
  const size_t hq = (size_t)c.n_q_heads * c.head_dim;
  L.T_alloc = (int)T;
  L.T_canvas = (int)Tc;
  L.P_alloc = (int)P;
  L.ks_r = router_splits(c);
  L.n_vt = c.vocab / 256;
  long long er = 0;
  for (int b = 1; b <= batch; ++b)
    er = std::max(er, (long long)esum_splits(c, b * DG_CANVAS, num_sms) * b * DG_CANVAS);
  L.epart_rows = er;
  L.err = take(64);
  L.flags = take(std::max<size_t>(batch, 64));
  L.x = take(T * d * 4);
  L.xn = take(T * d * 2);
  {
    const int qkv_rows = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim;
    size_t rq = 0, ro = 0;
    for (int tt = DG_CANVAS; tt <= (int)T; tt += DG_CANVAS) {
      rq = std::max(rq, (size_t)proj_splits((qkv_rows + 127) / 128, tt, c.d_model / 64, num_sms) * tt);
      ro = std::max(ro, (size_t)proj_splits((c.d_model + 127) / 128, tt, (int)hq / 64, num_sms, DG_O_SPLITS) * tt);
    }
    L.qkv = DG_QKV_CLUSTER ? 0 : take(rq * qkv_rows * 4);
    L.opart = DG_O_CLUSTER ? 0 : take(ro * d * 4);
  }
  L.q = take(T * hq * 2);
  L.attn = take(T * hq * 2);
  L.rpart = take((size_t)(DG_ROUTER_CLUSTER ? 1 : L.ks_r) * T * E * 4);  // router logits (or split partials)
  L.rbar = take(64);
  L.rfill = take(2 * E * 4);
  L.off = take((E + 1) * 4);
  L.choff = take((E + 1) * 4);
  L.perm = take(P * 4);
  L.inv = take(P * 4);
  L.wperm = take(P * 4);
  L.xperm = take(P * d * 2);
  L.hperm = take(P * (size_t)c.d_ff * 2);
  L.yperm = take(P * d * 4);
  L.logits = take(Tc * V * 2);
  const size_t nvp = Tc * (size_t)L.n_vt * 4;
  L.vp_m = take(nvp); L.vp_z = take(nvp); L.vp_s = take(nvp); L.vp_av = take(nvp);
  L.vp_ai = take(nvp); L.vp_gv = take(nvp); L.vp_gi = take(nvp);
  L.st_m = take(Tc * 4); L.st_iz = take(Tc * 4); L.st_h = take(Tc * 4); L.st_pmax = take(Tc * 4);
  L.st_amax = take(Tc * 4); L.st_samp = take(Tc * 4);
  L.tok = take(T * 4);
  L.xnc = take(Tc * d * 2);  // canvas rows of the normed stream after a fused append pass
  L.rope = take(T * (c.head_dim / 2) * 16);  // (cos, sin) of up to T positions of a pass
  L.stepdev = take(sizeof(StepDev));
  L.dstat = take((size_t)c.n_layers * 4);  // distinct experts per layer, summed over passes
  L.dep = take((P / 16 + E + 1) * 4);       // the fused expert kernel's chunk counters (chunks of >= 16 slots)
  L.probs = c.self_cond ? take(Tc * V * 2) : 0;
  L.epart = c.self_cond ? take((size_t)er * d * 4) : 0;
  L.total = off;
  return L;
}

// ---------------------------------------------------------------------------
// TMA tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// K-major bf16 matrix [rows, K] (row stride K elements), box 64 x box_rows,
// 128-byte swizzle.
dg_status make_tmap(CUtensorMap* m, const void* base, long long K, long long rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (((uintptr_t)base & 15) || K % 64 || rows < 1)
    return fail(DG_ERR_INVALID_ARG, "tensor map: bad base/K/rows (%p, %lld, %lld)", base, K, rows);
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DG_OK;
}

// General 2-D bf16 tensor map: `rows` rows of `inner` elements, `stride_bytes`
// apart; box box_inner x box_rows with the 128-byte swizzle (box_inner = 64).
// Elements past `inner` or `rows` read as zero.
dg_status make_tmap_2d(CUtensorMap* m, const void* base, long long inner, long long rows, long long stride_bytes,
                       int box_inner, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (((uintptr_t)base & 15) || inner < 1 || rows < 1 || stride_bytes % 16 || box_inner * 2 != 128 ||
      box_rows < 1 || box_rows > 256)
    return fail(DG_ERR_INVALID_ARG, "tensor map: bad base/extent/stride (%p, %lld, %lld, %lld)", base, inner, rows,
                stride_bytes);
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)stride_bytes};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DG_OK;
}

// fp32 tensor [slices][rows][inner] for tensor stores of 32 x 32 boxes with
// the 128-byte swizzle (boxes reaching past `rows` or `inner` are clipped).
dg_status make_tmap_f32_store(CUtensorMap* m, void* base, long long inner, long long rows, long long slices) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (((uintptr_t)base & 15) || inner < 1 || (inner * 4) % 16 || rows < 1 || slices < 1)
    return fail(DG_ERR_INVALID_ARG, "tensor map: bad fp32 store tensor (%p, %lld, %lld, %lld)", base, inner, rows,
                slices);
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)slices};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 4, (cuuint64_t)(inner * rows * 4)};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DG_OK;
}

// B operand of a GEMM: three tensor maps of the same matrix with boxes of 16,
// min(64, bn) and bn rows (each at most the matrix's rows).
struct BOperand {
  BMaps maps;
  int rows[3];
};

dg_status make_bop(BOperand* b, const void* base, long long K, long long rows, int bn) {
  const int want[3] = {16, std::min(64, bn), bn};
  for (int i = 0; i < 3; ++i) {
    b->rows[i] = (int)std::min<long long>(want[i], rows);
    DG_TRY(make_tmap(&b->maps.m[i], base, K, rows, b->rows[i]));
  }
  return DG_OK;
}

// B maps of a pair schedule: each CTA of a pair copies half of a unit's rows.
dg_status make_bop_half(BOperand* b, const void* base, long long K, long long rows, int bn) {
  const int want[3] = {8, std::min(32, bn / 2), bn / 2};
  for (int i = 0; i < 3; ++i) {
    b->rows[i] = (int)std::min<long long>(want[i], rows);
    DG_TRY(make_tmap(&b->maps.m[i], base, K, rows, b->rows[i]));
  }
  return DG_OK;
}

// cudaFuncSetAttribute applies to the kernel in the current device's context:
// set each (kernel, device) once, the first time a launch on that device
// needs it.
dg_status set_smem_attr(const void* fn, int bytes, bool max_carveout) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  DG_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({fn, dev})) return DG_OK;
  DG_CUDA(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  if (max_carveout) DG_CUDA(cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
  done.insert({fn, dev});
  return DG_OK;
}

int device_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

template <class Epi>
dg_status run_gemm(const CUtensorMap& ta, const BOperand& tb, GemmPlan p, const Epi& epi, int num_sms,
                   cudaStream_t st, long long* launches = nullptr) {
  if (p.bn < 16 || p.bn > 256 || (p.bn & (p.bn - 1)) || p.K % 64 || p.K < 64)
    return fail(DG_ERR_INVALID_ARG, "gemm plan: bn %d K %d", p.bn, p.K);
  if (p.group_off && (p.n_groups < 1 || p.n_groups > kGemmMaxGroups))
    return fail(DG_ERR_INVALID_ARG, "gemm plan: %d groups (1..%d)", p.n_groups, kGemmMaxGroups);
  if (p.mt != 1 && (p.mt != 2 || p.group_off))
    return fail(DG_ERR_INVALID_ARG, "gemm plan: %d A tiles per unit", p.mt);
  for (int i = 0; i < 3; ++i) {
    if (tb.rows[i] < 1 || tb.rows[i] > p.bn || (i && tb.rows[i] < tb.rows[i - 1]))
      return fail(DG_ERR_INVALID_ARG, "gemm plan: B box rows %d of bn %d", tb.rows[i], p.bn);
    p.b_rows[i] = tb.rows[i];
  }
  DG_TRY(set_smem_attr((const void*)gemm_tc_kernel<Epi>, (int)(227 * 1024 - kGemmStaticSmem), true));
  const int ctas = gemm_ctas_per_sm(p.bn, p.mt);
  const int stages = gemm_pick_stages(p.bn, ctas, 8, p.mt);
  const size_t smem = gemm_smem_bytes(p.bn, stages, p.mt);
  long long units;  // grouped: known only on the device; persistent CTAs
  if (p.group_off) units = (long long)ctas * num_sms;
  else units = (long long)((p.m_tiles + p.mt - 1) / p.mt) * ((p.n_total + p.bn - 1) / p.bn) * p.k_splits;
  if (units <= 0) return DG_OK;
  if (p.cluster_k <= 1) {
    p.cluster_k = 0;
    const int grid = (int)std::min<long long>(units, (long long)ctas * num_sms);
    DG_CUDA(Launch(dim3(grid), dim3(gemm_threads<Epi>()), smem, st)(gemm_tc_kernel<Epi>, ta, tb.maps, p, epi,
                                                                       stages));
  } else {
    // one unit per CTA; the k splits of a tile are consecutive units and one
    // cluster; their accumulators are staged in the stage ring ([128][bn + 4] fp32)
    if (p.group_off || p.mt != 1 || p.cluster_k != p.k_splits || p.cluster_k > 8)
      return fail(DG_ERR_INVALID_ARG, "gemm plan: cluster of %d k splits (dense, one A tile, at most 8)",
                  p.cluster_k);
    if ((size_t)stages * ((size_t)kATileBytes + (size_t)p.bn * 128) < (size_t)128 * (p.bn + 4) * 4)
      return fail(DG_ERR_INVALID_ARG, "gemm plan: the stage ring cannot hold a %d-column accumulator", p.bn);
    DG_CUDA(Launch(dim3((unsigned)units), dim3(gemm_threads<Epi>()), smem, st)
                .cluster((unsigned)p.cluster_k, 1, 1)
                .policy(DG_CLUSTER_POLICY ? cudaClusterSchedulingPolicyLoadBalancing
                                          : cudaClusterSchedulingPolicySpread)(gemm_tc_kernel<Epi>, ta, tb.maps, p,
                                                                               epi, stages));
  }
  if (launches) ++*launches;
  return DG_OK;
}

// The grouped schedule on 2-CTA clusters (see gemm_pair.cuh); tb from make_bop_half.
template <class Epi>
dg_status run_gemm_pair(const CUtensorMap& ta, const BOperand& tb, GemmPlan p, const Epi& epi, int num_sms,
                        cudaStream_t st, long long* launches = nullptr) {
  if ((p.group_off && (p.n_groups < 1 || p.n_groups > kGemmMaxGroups || p.k_splits != 1)) || p.mt != 1 ||
      p.k_splits < 1 || p.k_splits > p.K / 64)
    return fail(DG_ERR_INVALID_ARG, "pair gemm: %d groups, %d A tiles, %d k splits", p.n_groups, p.mt, p.k_splits);
  if (p.bn < 16 || p.bn > 256 || (p.bn & (p.bn - 1)) || p.K % 64 || p.K < 64)
    return fail(DG_ERR_INVALID_ARG, "pair gemm plan: bn %d K %d", p.bn, p.K);
  for (int i = 0; i < 3; ++i) {
    if (tb.rows[i] < 1 || (i && tb.rows[i] < tb.rows[i - 1]) || tb.rows[i] > p.bn / 2)
      return fail(DG_ERR_INVALID_ARG, "pair gemm plan: B box rows %d of bn %d", tb.rows[i], p.bn);
    p.b_rows[i] = tb.rows[i];
  }
  DG_TRY(set_smem_attr((const void*)gemm_pair_kernel<Epi>, (int)(227 * 1024 - kGemmStaticSmem), true));
  const int stages = gemm_pair_stages(p.bn);
  const size_t smem = gemm_pair_smem_bytes(p.bn, stages);
  const unsigned grid = (unsigned)(2 * (num_sms / 2) * gemm_pair_ctas_per_sm(p.bn));  // whole pairs
  DG_CUDA(Launch(dim3(grid), dim3(gemm_threads<Epi>()), smem, st).cluster(2, 1, 1)(gemm_pair_kernel<Epi>, ta,
                                                                                    tb.maps, p, epi, stages));
  if (launches) ++*launches;
  return DG_OK;
}

// Both grouped expert products in one launch on 2-CTA clusters (moe_pair.cuh);
// tb1 / tb2 from make_bop_half.
template <class EpiU, class EpiD>
dg_status run_moe_pair(const CUtensorMap& ta1, const BOperand& tb1, const CUtensorMap& ta2, const BOperand& tb2,
                       MoePlan mp, const EpiU& e1, const EpiD& e2, int num_sms, cudaStream_t st,
                       long long* launches = nullptr) {
  GemmPlan* ps[2] = {&mp.up, &mp.down};
  const BOperand* tbs[2] = {&tb1, &tb2};
  for (int q = 0; q < 2; ++q) {
    GemmPlan& p = *ps[q];
    if (!p.group_off || p.n_groups < 1 || p.n_groups > kGemmMaxGroups || p.mt != 1 || p.k_splits != 1 ||
        p.bn < 16 || p.bn > 128 || (p.bn & (p.bn - 1)) || p.K % 64 || p.K < 64)
      return fail(DG_ERR_INVALID_ARG, "expert kernel plan %d: groups %d bn %d K %d", q, p.n_groups, p.bn, p.K);
    for (int i = 0; i < 3; ++i) {
      if (tbs[q]->rows[i] < 1 || (i && tbs[q]->rows[i] < tbs[q]->rows[i - 1]) || tbs[q]->rows[i] > p.bn / 2)
        return fail(DG_ERR_INVALID_ARG, "expert kernel plan %d: B box rows %d of bn %d", q, tbs[q]->rows[i], p.bn);
      p.b_rows[i] = tbs[q]->rows[i];
    }
  }
  if (mp.up.bn != mp.down.bn || mp.up.n_groups != mp.down.n_groups || mp.up.group_off != mp.down.group_off ||
      mp.up.chunk_off != mp.down.chunk_off || !mp.dep)
    return fail(DG_ERR_INVALID_ARG, "expert kernel: the two products must share groups and chunks");
  DG_TRY(set_smem_attr((const void*)moe_pair_kernel<EpiU, EpiD>, (int)(227 * 1024 - kGemmStaticSmem), true));
  const int stages = gemm_pair_stages(mp.up.bn);
  const size_t smem = gemm_pair_smem_bytes(mp.up.bn, stages);
  const unsigned grid = (unsigned)(2 * (num_sms / 2) * gemm_pair_ctas_per_sm(mp.up.bn));  // whole pairs
  DG_CUDA(Launch(dim3(grid), dim3(gemm_threads<EpiU>()), smem, st).cluster(2, 1, 1)(
      moe_pair_kernel<EpiU, EpiD>, ta1, tb1.maps, ta2, tb2.maps, mp, e1, e2, stages));
  if (launches) ++*launches;
  return DG_OK;
}

GemmPlan dense_plan(int K, int a_rows, int n_total, int bn, int k_splits, int* err) {
  GemmPlan p{};
  p.K = K;
  p.a_rows = a_rows;
  p.m_tiles = (a_rows + 127) / 128;
  p.n_total = n_total;
  p.bn = bn;
  p.k_splits = k_splits;
  p.n_fast = 1;
  p.group_off = nullptr;
  p.mt = 1;
  p.err = err;
  return p;
}

GemmPlan grouped_plan(int K, int rows_per_group, const int* off, const int* chunk_off, int n_groups, int bn,
                      int* err) {
  GemmPlan p{};
  p.chunk_off = chunk_off;
  p.K = K;
  p.a_rows = rows_per_group;
  p.m_tiles = (rows_per_group + 127) / 128;
  p.n_total = 0;
  p.bn = bn;
  p.k_splits = 1;
  p.group_off = off;
  p.n_groups = n_groups;
  p.a_rows_per_group = rows_per_group;
  p.mt = 1;
  p.err = err;
  return p;
}

int token_bn(int T) { return std::min(256, std::max(16, next_pow2(T))); }

// Token columns per unit of a weight-stationary dense GEMM: the largest tile
// (up to 256) that still gives about one unit per SM, so small batches spread
// the weight stream over the whole GPU (tiles re-read their weights from L2).
int dense_bn(int m_tiles, int T, int num_sms) {
  int bn = token_bn(T);
  while (bn > 16 && (long long)m_tiles * ((T + bn - 1) / bn) < (3 * num_sms) / 4) bn >>= 1;
  return bn;
}

}  // namespace

// ============================================================================
struct dg_ctx {
  // measurement hooks: launch counter and per-class CUDA-event brackets
  bool prof = false;
  long long n_launch = 0;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<std::pair<int, int>> prof_recs;  // (class, index of the start event)
  int ev_used = 0;
  int prof_begin(int kind, cudaStream_t st) {
    if (!prof || prof_recs.size() >= 65536) return -1;
    while ((int)ev_pool.size() < ev_used + 2) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return -1;
      ev_pool.push_back(e);
    }
    const int i = ev_used;
    ev_used += 2;
    cudaEventRecord(ev_pool[i], st);
    prof_recs.push_back({kind, i});
    return i;
  }
  void prof_end(int i, cudaStream_t st) {
    if (i >= 0) cudaEventRecord(ev_pool[i + 1], st);
  }
  // cached CUDA graph of one round (dg_denoise_step_graph)
  struct GraphKey {
    dg_kv kv;
    dg_canvas cv;
    dg_step_out out;
    int32_t topk;   // the a8 form the graph was captured with
  };
  bool g_valid = false;
  GraphKey g_key;
  cudaGraph_t g_graph = nullptr;
  cudaGraphExec_t g_exec = nullptr;
  cudaGraphNode_t g_param_node = nullptr;
  cudaStream_t g_stream = nullptr;
  long long g_kernels = 0;  // kernels launched by one replay
  void drop_graph() {
    if (g_exec) cudaGraphExecDestroy(g_exec);
    if (g_graph) cudaGraphDestroy(g_graph);
    g_exec = nullptr;
    g_graph = nullptr;
    g_param_node = nullptr;
    g_valid = false;
  }
  ~dg_ctx() {
    drop_graph();
    if (g_stream) cudaStreamDestroy(g_stream);
    for (cudaEvent_t e : ev_pool) cudaEventDestroy(e);
  }
  dg_model_config cfg;
  const uint16_t* w;
  uint8_t* ws;
  size_t ws_bytes;
  int batch_max;
  int num_sms;
  WLayout wl;
  WsLayout L;
  template <class T>
  T* at(size_t off) const { return reinterpret_cast<T*>(ws + off); }
  const uint16_t* wp(size_t off) const { return w + off; }
  int* err() const { return at<int>(L.err); }
};

// Brackets the launches of one profiled class with CUDA events (no-op when
// profiling is off).
struct ProfScope {
  dg_ctx* c;
  cudaStream_t st;
  int idx;
  ProfScope(dg_ctx* c_, int kind, cudaStream_t s) : c(c_), st(s), idx(c_->prof_begin(kind, s)) {}
  ~ProfScope() { c->prof_end(idx, st); }
};
#define CNT(c) (++(c)->n_launch)

extern "C" size_t dg_weights_bytes(const dg_model_config* cfg) {
  char why[256];
  if (!cfg_ok(cfg, why, sizeof why)) { fail(DG_ERR_INVALID_ARG, "%s", why); return 0; }
  return weight_layout(*cfg).total * 2;
}

extern "C" size_t dg_kv_bytes(const dg_model_config* cfg, int32_t batch, int32_t c_max) {
  char why[256];
  if (!cfg_ok(cfg, why, sizeof why) || batch < 1 || c_max < 8 || c_max % 8) {
    fail(DG_ERR_INVALID_ARG, "bad kv size query (c_max must be a positive multiple of 8)");
    return 0;
  }
  return (size_t)cfg->n_layers * batch * cfg->n_kv_heads * c_max * cfg->head_dim * 2;
}

extern "C" size_t dg_workspace_bytes_ex(const dg_model_config* cfg, int32_t batch, int32_t prefill_tokens) {
  char why[256];
  if (!cfg_ok(cfg, why, sizeof why) || batch < 1 || prefill_tokens < 0 || prefill_tokens > (1 << 20)) {
    fail(DG_ERR_INVALID_ARG, "bad workspace query");
    return 0;
  }
  return ws_layout(*cfg, batch, device_sms(), prefill_tokens).total;
}

extern "C" size_t dg_workspace_bytes(const dg_model_config* cfg, int32_t batch) {
  return dg_workspace_bytes_ex(cfg, batch, 0);
}

extern "C" dg_status dg_model_init_random(const dg_model_config* cfg, uint64_t seed, const float* kind_std,
                                          void* d_weights, void* stream) {
  char why[256];
  if (!cfg_ok(cfg, why, sizeof why)) return fail(DG_ERR_INVALID_ARG, "%s", why);
  if (!d_weights || ((uintptr_t)d_weights & 255)) return fail(DG_ERR_INVALID_ARG, "weights must be 256-byte aligned");
  const dg_model_config& c = *cfg;
  const WLayout wl = weight_layout(c);
  uint16_t* W = (uint16_t*)d_weights;
  cudaStream_t st = (cudaStream_t)stream;
  auto sd = [&](int kind) -> double {
    return (kind_std && kind_std[kind] > 0.f) ? (double)kind_std[kind] : 0.02;
  };
  auto fill = [&](uint16_t* dst, long long rows, long long cols, long long sr, long long sc, uint32_t tid,
                  int kind) -> dg_status {
    int r = synth_fill_bf16_device(dst, 0, rows, cols, sr, sc, seed, tid, sd(kind), st);
    if (r) return fail(DG_ERR_CUDA, "weight init: %s", cudaGetErrorString((cudaError_t)r));
    return DG_OK;
  };
  auto fill_rows = [&](uint16_t* dst, long long row0, long long rows, long long cols, long long sr, long long sc,
                       uint32_t tid, int kind) -> dg_status {
    int r = synth_fill_bf16_device(dst, row0, rows, cols, sr, sc, seed, tid, sd(kind), st);
    if (r) return fail(DG_ERR_CUDA, "weight init: %s", cudaGetErrorString((cudaError_t)r));
    return DG_OK;
  };
  auto ones = [&](uint16_t* dst, long long n) -> dg_status {
    fill_u16_kernel<<<(unsigned)std::min<long long>((n + 255) / 256, 4096), 256, 0, st>>>(dst, n, 0x3F80);
    DG_CUDA(cudaGetLastError());
    return DG_OK;
  };
  const long long d = c.d_model, V = c.vocab, hd = c.head_dim, E = c.n_experts, f = c.d_ff;
  DG_CUDA(cudaMemsetAsync(W, 0, wl.total * 2, st));
  DG_TRY(fill(W + wl.emb, V, d, d, 1, SYNTH_KIND_EMB, SYNTH_KIND_EMB));
  DG_TRY(fill(W + wl.embT, V, d, 1, V, SYNTH_KIND_EMB, SYNTH_KIND_EMB));  // transposed copy
  DG_TRY(fill(W + wl.lm, V, d, d, 1, SYNTH_KIND_LM, SYNTH_KIND_LM));
  if (c.self_cond) DG_TRY(fill(W + wl.sc, d, d, d, 1, SYNTH_KIND_SC, SYNTH_KIND_SC));
  DG_TRY(ones(W + wl.g_final, d));
  for (int l = 0; l < c.n_layers; ++l) {
    const LayerW& L = wl.layers[l];
    uint16_t* qkv = W + L.wqkv;
    // q and k heads: rotation pairs (j, j + hd/2) of a head in adjacent physical
    // rows 2j, 2j + 1 (the QKV epilogue rotates a pair across two lanes)
    for (int h = 0; h < c.n_q_heads + c.n_kv_heads; ++h) {
      const bool is_q = h < c.n_q_heads;
      const int hl = is_q ? h : h - c.n_q_heads;
      const int kind = is_q ? SYNTH_KIND_WQ : SYNTH_KIND_WK;
      for (int hf = 0; hf < 2; ++hf)
        DG_TRY(fill_rows(qkv + ((long long)h * hd + hf) * d, (long long)hl * hd + hf * (hd / 2), hd / 2, d, 2 * d, 1,
                         synth_layer_tid(l, kind), kind));
    }
    DG_TRY(fill(qkv + (long long)(c.n_q_heads + c.n_kv_heads) * hd * d, c.n_kv_heads * hd, d, d, 1,
                synth_layer_tid(l, SYNTH_KIND_WV), SYNTH_KIND_WV));
    DG_TRY(fill(W + L.wo, d, c.n_q_heads * hd, c.n_q_heads * hd, 1, synth_layer_tid(l, SYNTH_KIND_WO),
                SYNTH_KIND_WO));
    DG_TRY(fill(W + L.wr, E, d, d, 1, synth_layer_tid(l, SYNTH_KIND_WR), SYNTH_KIND_WR));
    // gate row j of expert e -> physical row 2(e f + j), up row -> 2(e f + j) + 1
    DG_TRY(fill(W + L.wgu, E * f, d, 2 * d, 1, synth_layer_tid(l, SYNTH_KIND_WG), SYNTH_KIND_WG));
    DG_TRY(fill(W + L.wgu + d, E * f, d, 2 * d, 1, synth_layer_tid(l, SYNTH_KIND_WU), SYNTH_KIND_WU));
    DG_TRY(fill(W + L.wd, E * d, f, f, 1, synth_layer_tid(l, SYNTH_KIND_WD), SYNTH_KIND_WD));
    DG_TRY(ones(W + L.g_attn, d));
    DG_TRY(ones(W + L.g_moe, d));
  }
  return DG_OK;
}

extern "C" dg_status dg_context_create(const dg_model_config* cfg, const void* d_weights, void* d_workspace,
                                       size_t ws_bytes, int32_t batch, dg_ctx** out) {
  return dg_context_create_ex(cfg, d_weights, d_workspace, ws_bytes, batch, 0, out);
}

extern "C" dg_status dg_context_create_ex(const dg_model_config* cfg, const void* d_weights, void* d_workspace,
                                          size_t ws_bytes, int32_t batch, int32_t prefill_tokens, dg_ctx** out) {
  if (!out) return fail(DG_ERR_INVALID_ARG, "out is null");
  if (prefill_tokens < 0 || prefill_tokens > (1 << 20)) return fail(DG_ERR_INVALID_ARG, "prefill_tokens outside [0, 2^20]");
  *out = nullptr;
  char why[256];
  if (!cfg_ok(cfg, why, sizeof why)) return fail(DG_ERR_INVALID_ARG, "%s", why);
  if (batch < 1 || batch > 64) return fail(DG_ERR_INVALID_ARG, "batch must be in [1, 64]");
  if (!d_weights || !d_workspace || ((uintptr_t)d_workspace & 255) || ((uintptr_t)d_weights & 255))
    return fail(DG_ERR_INVALID_ARG, "weights and workspace must be non-null and 256-byte aligned");
  dg_ctx* c = new (std::nothrow) dg_ctx();
  if (!c) return fail(DG_ERR_INVALID_ARG, "host allocation failed");
  c->cfg = *cfg;
  c->w = (const uint16_t*)d_weights;
  c->ws = (uint8_t*)d_workspace;
  c->ws_bytes = ws_bytes;
  c->batch_max = batch;
  c->num_sms = device_sms();
  c->wl = weight_layout(*cfg);
  c->L = ws_layout(*cfg, batch, c->num_sms, prefill_tokens);
  if (ws_bytes < c->L.total) {
    size_t need = c->L.total;
    delete c;
    return fail(DG_ERR_WORKSPACE, "workspace too small: %zu < %zu", ws_bytes, need);
  }
  cudaError_t e = cudaMemset(c->ws + c->L.err, 0, 64);
  if (e == cudaSuccess) e = cudaMemset(c->ws + c->L.rbar, 0, 64);
  if (e == cudaSuccess) e = cudaMemset(c->ws + c->L.rfill, 0, (size_t)cfg->n_experts * 8);
  if (e != cudaSuccess) {
    delete c;
    return fail(DG_ERR_CUDA, "cudaMemset: %s", cudaGetErrorString(e));
  }
  *out = c;
  return DG_OK;
}

extern "C" void dg_context_destroy(dg_ctx* ctx) { delete ctx; }

// ---------------------------------------------------------------------------
// Attention of one pass on the tensor cores: q packed [B][Hkv][nq][G][hd],
// K cache [B][Hkv][c_max][hd], V^T cache [B][Hkv][hd][c_max]; splits > 1
// writes per-split partials and merges them (fixed split order) into out.

// With `cluster`, the key splits of a tile run as one thread-block cluster and
// merge through distributed shared memory (part_o / part_ml unused); without
// it they write partials to part_o / part_ml and a second kernel merges them.
template <int HD>
static dg_status launch_attn(dim3 grid, int splits, bool cluster, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, const CUtensorMap& to, const AttnTcParams& ap, cudaStream_t st) {
  DG_TRY(set_smem_attr((const void*)attn_tc_kernel<HD>, (int)AttnTcShape<HD>::SMEM, false));
  Launch l(grid, dim3(kAttnThreads), AttnTcShape<HD>::SMEM, st);
  if (cluster && splits > 1) l.cluster(1, 1, (unsigned)splits);
  DG_CUDA(l(attn_tc_kernel<HD>, tq, tk, tv, to, ap));
  return DG_OK;
}

static dg_status run_attention(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, uint16_t* out,
                               float* part_o, float* part_ml, int B, int nq, int L0, int c_max, int Hq, int Hkv,
                               int hd, int causal_n, int splits, bool cluster, int* err, cudaStream_t st,
                               long long* launches) {
  if (c_max % 8) return fail(DG_ERR_INVALID_ARG, "c_max %d is not a multiple of 8", c_max);
  if (splits > kMaxAttnSplits) return fail(DG_ERR_INVALID_ARG, "%d key splits (at most %d)", splits, kMaxAttnSplits);
  if (splits > 1 && !cluster && (!part_o || !part_ml)) return fail(DG_ERR_INVALID_ARG, "split buffers are null");
  const int G = Hq / Hkv;
  CUtensorMap tq, tk, tv;
  DG_TRY(make_tmap_2d(&tq, q, hd, (long long)B * Hkv * nq * G, (long long)hd * 2, 64, kAttnRows));
  DG_TRY(make_tmap_2d(&tk, kc, hd, (long long)B * Hkv * c_max, (long long)hd * 2, 64, kAttnKeys));
  DG_TRY(make_tmap_2d(&tv, vc, L0 + nq, (long long)B * Hkv * hd, (long long)c_max * 2, 64, hd));
  CUtensorMap to;
  memset(&to, 0, sizeof to);
  const bool merge_in_cluster = cluster && splits > 1;
  if (splits > 1 && !merge_in_cluster)
    DG_TRY(make_tmap_f32_store(&to, part_o, hd, (long long)G * nq, (long long)splits * B * Hkv));
  AttnTcParams ap{out, part_o, part_ml, B, nq, L0, c_max, Hq, Hkv, splits, causal_n,
                  (float)(1.4426950408889634 / sqrt((double)hd)), err, merge_in_cluster ? 1 : 0};
  dim3 grid((G * nq + kAttnRows - 1) / kAttnRows, Hkv, B * splits);
  switch (hd) {
    case 32: DG_TRY(launch_attn<32>(grid, splits, merge_in_cluster, tq, tk, tv, to, ap, st)); break;
    case 64: DG_TRY(launch_attn<64>(grid, splits, merge_in_cluster, tq, tk, tv, to, ap, st)); break;
    case 128: DG_TRY(launch_attn<128>(grid, splits, merge_in_cluster, tq, tk, tv, to, ap, st)); break;
    case 176: DG_TRY(launch_attn<176>(grid, splits, merge_in_cluster, tq, tk, tv, to, ap, st)); break;
    default: return fail(DG_ERR_UNSUPPORTED, "head_dim %d", hd);
  }
  if (launches) ++*launches;
  if (splits > 1 && !merge_in_cluster) {
    const long long rows = (long long)B * Hq * nq;
    const unsigned cgrid = (unsigned)((rows * 32 + 255) / 256);
    if (splits <= 4)
      DG_CUDA(Launch(dim3(cgrid), dim3(256), 0, st)(attn_combine_kernel<4>, part_o, part_ml, out, splits, B, Hq, Hkv, nq, hd));
    else
      DG_CUDA(Launch(dim3(cgrid), dim3(256), 0, st)(attn_combine_kernel<8>, part_o, part_ml, out, splits, B, Hq, Hkv, nq, hd));
    DG_CUDA(cudaGetLastError());
    if (launches) ++*launches;
  }
  return DG_OK;
}

// Key splits of a pass: enough CTAs to cover the SMs once (at most 8 splits,
// at most one split per 64-key tile).
static int attn_splits(int B, int nq, int L0, int Hq, int Hkv, int num_sms, int cap_rows) {
  const int base = ((Hq / Hkv) * nq + kAttnRows - 1) / kAttnRows * Hkv * B;
  const int n_kt = (L0 + nq + kAttnKeys - 1) / kAttnKeys;
  int s = std::max(1, std::min(num_sms / std::max(1, base), kMaxAttnSplits));
  s = std::min(s, n_kt);
  while (s > 1 && (long long)s * B > cap_rows) --s;
  return s;
}

// ============================================================================
// one pass of the transformer layers over T = B * nq tokens at positions
// L0 .. L0 + nq - 1 (x already holds the embedded inputs)
static dg_status forward_layers(dg_ctx* c, const dg_kv* kv, int B, int nq, int L0, int causal_n,
                                int32_t* dbg_idx, float* dbg_w, float* dbg_logits, float* dbg_hidden,
                                float* dbg_hidden_attn, cudaStream_t st) {
  const dg_model_config& m = c->cfg;
  const WsLayout& L = c->L;
  const int T = B * nq, d = m.d_model, hd = m.head_dim, Hq = m.n_q_heads, Hkv = m.n_kv_heads;
  const int E = m.n_experts, k = m.top_k, f = m.d_ff, P = T * k;
  const int qkv_rows = c->wl.qkv_rows;
  int* err = c->err();
  float* x = c->at<float>(L.x);
  uint16_t* xn = c->at<uint16_t>(L.xn);
  // token rows per grouped unit: 128 (256 for large batches).  Routing can be
  // very uneven; one unit per 128 tokens of an expert keeps the number of times
  // a weight tile is read small while the units of one tile run side by side.
  const int bnG = DG_GROUPED_BN ? DG_GROUPED_BN : (P / E > 64 ? 256 : 128);
  const size_t kv_layer = (size_t)kv->batch * Hkv * kv->c_max * hd;

  BOperand t_xperm, t_hperm;
  DG_TRY(make_bop(&t_xperm, c->at<uint16_t>(L.xperm), d, L.P_alloc, bnG));
  DG_TRY(make_bop(&t_hperm, c->at<uint16_t>(L.hperm), f, L.P_alloc, bnG));
  // grouped products of at most 128 tokens per chunk run on CTA pairs (two
  // pairs per SM pair); 256-token chunks keep one CTA per tile
  const bool pair = bnG <= 128 || DG_GROUPED_BN == 256;
  BOperand h_xperm{}, h_hperm{};
  if (pair) {
    DG_TRY(make_bop_half(&h_xperm, c->at<uint16_t>(L.xperm), d, L.P_alloc, bnG));
    DG_TRY(make_bop_half(&h_hperm, c->at<uint16_t>(L.hperm), f, L.P_alloc, bnG));
  }

  // cos/sin of this pass's positions, shared by all layers
  {
    const int n = nq * (hd / 2);
    DG_CUDA(Launch(dim3((n + 255) / 256), dim3(256), 0, st)(rope_table_kernel, c->at<double2>(L.rope), nq, L0, hd / 2, hd,
                                                       (double)m.rope_theta));
    CNT(c);
  }

  // split-k of the two dense projections (partials summed by their consumers)
  const int dense_bn_x = proj_bn(T);
  const int ks_qkv = proj_splits((qkv_rows + 127) / 128, T, d / 64, c->num_sms);
  const int ks_o = proj_splits((d + 127) / 128, T, Hq * hd / 64, c->num_sms, DG_O_SPLITS);

  // attention key splits (merged inside each split cluster)
  const int splits = attn_splits(B, nq, L0, Hq, Hkv, c->num_sms, 1 << 30);

  for (int l = 0; l < m.n_layers; ++l) {
    const LayerW& W = c->wl.layers[l];
    uint16_t* kc = (uint16_t*)kv->k + (size_t)l * kv_layer;
    uint16_t* vc = (uint16_t*)kv->v + (size_t)l * kv_layer;

    // --- attention block (its RMSNorm ran at the end of the previous layer) ---
    NvtxRange nv_layer("dg.layer");  // the whole layer; its expert block nested
    if (l == 0) {
      DG_CUDA(Launch(dim3(T), dim3(256), 0, st)(rmsnorm_kernel<256>, x, c->wp(W.g_attn), xn, d, m.rms_eps));
      CNT(c);
    }
    {
      ProfScope ps_(c, DG_PROF_DENSE, st);
      CUtensorMap ta;
      BOperand tb;
      const int bn = dense_bn_x;
      DG_TRY(make_tmap(&ta, c->wp(W.wqkv), d, qkv_rows, 128));
      GemmPlan p = dense_plan(d, qkv_rows, T, bn, ks_qkv, err);
      p.a_hint = 1;
      const bool pair_qkv = DG_PROJ_PAIR && !DG_QKV_CLUSTER;
      if (pair_qkv) DG_TRY(make_bop_half(&tb, xn, d, L.T_alloc, bn));
      else          DG_TRY(make_bop(&tb, xn, d, L.T_alloc, bn));
      if (pair_qkv) {
        if (ks_qkv == 1) {
          EpiQKV e{c->at<double2>(L.rope), c->at<uint16_t>(L.q), kc, vc, nq, L0, kv->c_max, Hq, Hkv, hd};
          DG_TRY(run_gemm_pair(ta, tb, p, e, c->num_sms, st, &c->n_launch));
        } else {
          EpiStoreT e{c->at<float>(L.qkv), qkv_rows, (long long)T * qkv_rows, 0, nullptr, nullptr, 0, err};
          DG_TRY(run_gemm_pair(ta, tb, p, e, c->num_sms, st, &c->n_launch));
        }
      } else if (DG_QKV_CLUSTER || ks_qkv == 1) {
        p.cluster_k = ks_qkv;  // the k splits of a tile add up in their cluster
        EpiQKV e{c->at<double2>(L.rope), c->at<uint16_t>(L.q), kc, vc, nq, L0, kv->c_max, Hq, Hkv, hd};
        DG_TRY(run_gemm(ta, tb, p, e, c->num_sms, st, &c->n_launch));
      } else {
        EpiStoreT e{c->at<float>(L.qkv), qkv_rows, (long long)T * qkv_rows, 0, nullptr, nullptr, 0, err};
        DG_TRY(run_gemm(ta, tb, p, e, c->num_sms, st, &c->n_launch));
      }
    }
    if (!DG_QKV_CLUSTER && ks_qkv > 1) {
      const int v_blocks = (int)(((long long)T * Hkv * (hd / 4) + 255) / 256);
      RopeParams rp{c->at<float>(L.qkv), ks_qkv, (long long)T * qkv_rows, c->at<double2>(L.rope),
                    c->at<uint16_t>(L.q), kc, vc, T, nq, L0, kv->c_max, Hq, Hkv, hd, v_blocks};
      if (ks_qkv > kRopeMaxSplits) return fail(DG_ERR_UNSUPPORTED, "QKV split count %d", ks_qkv);
      const long long rot_threads = (long long)T * (Hq + Hkv) * (hd / 8);
      const int rot_blocks = (int)((rot_threads + 255) / 256);
      DG_CUDA(Launch(dim3(rot_blocks + v_blocks), dim3(256), 0, st)(rope_kv_kernel, rp));
      CNT(c);
    }
    {
      ProfScope ps_(c, DG_PROF_ATTENTION, st);
      DG_TRY(run_attention(c->at<uint16_t>(L.q), kc, vc, c->at<uint16_t>(L.attn), nullptr, nullptr, B, nq, L0,
                           kv->c_max, Hq, Hkv, hd, causal_n, splits, true, err, st, &c->n_launch));
    }
    {
      ProfScope ps_(c, DG_PROF_DENSE, st);
      CUtensorMap ta;
      BOperand tb;
      const int bn = dense_bn_x;
      DG_TRY(make_tmap(&ta, c->wp(W.wo), (long long)Hq * hd, d, 128));
      GemmPlan p = dense_plan(Hq * hd, d, T, bn, ks_o, err);
      p.a_hint = 1;
      const bool pair_o = DG_PROJ_PAIR && !DG_O_CLUSTER;
      if (pair_o) DG_TRY(make_bop_half(&tb, c->at<uint16_t>(L.attn), (long long)Hq * hd, L.T_alloc, bn));
      else        DG_TRY(make_bop(&tb, c->at<uint16_t>(L.attn), (long long)Hq * hd, L.T_alloc, bn));
      if (pair_o) {
        if (ks_o == 1) {
          EpiStoreT e{x, d, 0, 1, nullptr, nullptr, 0, err};  // residual add: x += attn W_o^T
          DG_TRY(run_gemm_pair(ta, tb, p, e, c->num_sms, st, &c->n_launch));
        } else {
          EpiStoreT e{c->at<float>(L.opart), d, (long long)T * d, 0, nullptr, nullptr, 0, err};
          DG_TRY(run_gemm_pair(ta, tb, p, e, c->num_sms, st, &c->n_launch));
        }
      } else if (DG_O_CLUSTER || ks_o == 1) {
        p.cluster_k = ks_o;
        EpiStoreT e{x, d, 0, 1, nullptr, nullptr, 0, err};  // residual add: x += attn W_o^T
        DG_TRY(run_gemm(ta, tb, p, e, c->num_sms, st, &c->n_launch));
      } else {
        EpiStoreT e{c->at<float>(L.opart), d, (long long)T * d, 0, nullptr, nullptr, 0, err};
        DG_TRY(run_gemm(ta, tb, p, e, c->num_sms, st, &c->n_launch));
      }
    }

    // --- mixture of experts block: residual add (split partials) + RMSNorm ---
    NvtxRange nv_moe("dg.layer.moe_block");
    {
      const bool parts = !(DG_O_CLUSTER || ks_o == 1);
      DG_CUDA(Launch(dim3(T), dim3(row_launch(d).threads), 0, st)(residual_norm_kernel<1>, x, parts ? c->at<float>(L.opart) : nullptr,
                                                                   parts ? ks_o : 0, (long long)T * d, d,
                                                                   c->wp(W.g_moe), xn, m.rms_eps));
    }
    CNT(c);
    if (dbg_hidden_attn)
      DG_CUDA(cudaMemcpyAsync(dbg_hidden_attn + (size_t)l * T * d, x, (size_t)T * d * 4,
                              cudaMemcpyDeviceToDevice, st));
    {
      ProfScope ps_(c, DG_PROF_DENSE, st);
      CUtensorMap ta;
      BOperand tb;
      const int bn = std::max(32, dense_bn((E + 127) / 128, T, c->num_sms / L.ks_r));
      DG_TRY(make_tmap(&ta, c->wp(W.wr), d, c->wl.wr_rows, 128));
      DG_TRY(make_bop(&tb, xn, d, L.T_alloc, bn));
      GemmPlan p = dense_plan(d, E, T, bn, L.ks_r, err);
      if (DG_ROUTER_CLUSTER) {
        p.cluster_k = L.ks_r;  // final router logits [T, E]
        EpiStoreT e{c->at<float>(L.rpart), E, 0, 0, nullptr, nullptr, 0, err};
        DG_TRY(run_gemm(ta, tb, p, e, c->num_sms, st, &c->n_launch));
      } else {
        EpiStoreT e{c->at<float>(L.rpart), E, (long long)T * E, 0, nullptr, nullptr, 0, err};
        DG_TRY(run_gemm(ta, tb, p, e, c->num_sms, st, &c->n_launch));
      }
    }
    {
      // top-k, counting sort by expert and row gather in one cooperative launch
      RouteParams rp;
      rp.part = c->at<float>(L.rpart);
      rp.xn = xn;
      rp.T = T; rp.E = E; rp.k = k; rp.d = d; rp.bn = bnG;
      rp.tpc = (T + c->num_sms - 1) / c->num_sms;
      rp.off = c->at<int>(L.off);
      rp.chunk_off = c->at<int>(L.choff);
      rp.perm = c->at<int>(L.perm);
      rp.inv = c->at<int>(L.inv);
      rp.w_perm = c->at<float>(L.wperm);
      rp.xperm = c->at<uint16_t>(L.xperm);
      rp.fill = c->at<int>(L.rfill);
      rp.bar = c->at<int>(L.rbar);
      // an appending pass records the routing of its canvas rows only
      rp.dbg_nq = causal_n > 0 && causal_n < nq ? nq : 0;
      rp.dbg_skip = rp.dbg_nq ? causal_n : 0;
      const size_t T_dbg = rp.dbg_nq ? (size_t)B * (nq - causal_n) : (size_t)T;
      rp.dbg_idx = dbg_idx ? dbg_idx + (size_t)l * T_dbg * k : nullptr;
      rp.dbg_w = dbg_w ? dbg_w + (size_t)l * T_dbg * k : nullptr;
      rp.dbg_logits = dbg_logits ? dbg_logits + (size_t)l * T_dbg * E : nullptr;
      rp.distinct = c->at<int>(L.dstat) + l;
      rp.dep = c->at<int>(L.dep);
      rp.dep_n = (int)(L.P_alloc / 16 + E + 1);
      rp.err = err;
      const int nb = (T + rp.tpc - 1) / rp.tpc;
      cudaLaunchConfig_t lc = {};
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeCooperative;
      at[0].val.cooperative = 1;
      lc.gridDim = dim3(nb);
      lc.blockDim = dim3(kRouteThreads);
      lc.dynamicSmemBytes = route_smem_bytes(rp.tpc, k, E);
      lc.stream = st;
      lc.attrs = at;
      lc.numAttrs = 1;
      const int ksr = DG_ROUTER_CLUSTER ? 1 : L.ks_r;
      if (ksr == 8)      DG_CUDA(cudaLaunchKernelEx(&lc, route_kernel<8>, rp));
      else if (ksr == 4) DG_CUDA(cudaLaunchKernelEx(&lc, route_kernel<4>, rp));
      else if (ksr == 1) DG_CUDA(cudaLaunchKernelEx(&lc, route_kernel<1>, rp));
      else return fail(DG_ERR_UNSUPPORTED, "router split count %d", ksr);
      CNT(c);
    }
    if (pair && DG_MOE_FUSED) {
      // gate/up + SwiGLU and down in one launch
      ProfScope ps_(c, DG_PROF_EXPERT_GATE_UP, st);
      CUtensorMap ta1, ta2;
      DG_TRY(make_tmap(&ta1, c->wp(W.wgu), d, (long long)E * 2 * f, 128));
      DG_TRY(make_tmap(&ta2, c->wp(W.wd), f, (long long)E * d, 128));
      MoePlan mp;
      mp.up = grouped_plan(d, 2 * f, c->at<int>(L.off), c->at<int>(L.choff), E, bnG, err);
      mp.down = grouped_plan(f, d, c->at<int>(L.off), c->at<int>(L.choff), E, bnG, err);
      mp.up.a_hint = mp.down.a_hint = 1;
      mp.up.b_hint = mp.down.b_hint = 2;
      mp.dep = c->at<int>(L.dep);
      EpiSwiGLU e1{c->at<uint16_t>(L.hperm), f};
      EpiDown e2{c->at<float>(L.yperm), d, c->at<float>(L.wperm)};
      DG_TRY(run_moe_pair(ta1, h_xperm, ta2, h_hperm, mp, e1, e2, c->num_sms, st, &c->n_launch));
    } else {
    {
      ProfScope ps_(c, DG_PROF_EXPERT_GATE_UP, st);
      CUtensorMap ta;
      DG_TRY(make_tmap(&ta, c->wp(W.wgu), d, (long long)E * 2 * f, 128));
      GemmPlan p = grouped_plan(d, 2 * f, c->at<int>(L.off), c->at<int>(L.choff), E, bnG, err);
      p.a_hint = 1;
      p.b_hint = 2;
      EpiSwiGLU e{c->at<uint16_t>(L.hperm), f};
      if (pair) DG_TRY(run_gemm_pair(ta, h_xperm, p, e, c->num_sms, st, &c->n_launch));
      else      DG_TRY(run_gemm(ta, t_xperm, p, e, c->num_sms, st, &c->n_launch));
    }
    {
      ProfScope ps_(c, DG_PROF_EXPERT_DOWN, st);
      CUtensorMap ta;
      DG_TRY(make_tmap(&ta, c->wp(W.wd), f, (long long)E * d, 128));
      GemmPlan p = grouped_plan(f, d, c->at<int>(L.off), c->at<int>(L.choff), E, bnG, err);
      p.a_hint = 1;
      p.b_hint = 2;
      EpiDown e{c->at<float>(L.yperm), d, c->at<float>(L.wperm)};
      if (pair) DG_TRY(run_gemm_pair(ta, h_hperm, p, e, c->num_sms, st, &c->n_launch));
      else      DG_TRY(run_gemm(ta, t_hperm, p, e, c->num_sms, st, &c->n_launch));
    }
    }
    // combine + residual, fused with the next RMSNorm (next layer's attention
    // norm, or the final norm before the LM head)
    {
      const uint16_t* g_next = l + 1 < m.n_layers ? c->wp(c->wl.layers[l + 1].g_attn) : c->wp(c->wl.g_final);
      // the next layer's QKV weights go to L2 during the combine
      const void* pf = l + 1 < m.n_layers ? (const void*)c->wp(c->wl.layers[l + 1].wqkv) : nullptr;
      // two float4s per thread: the eight expert rows per float4 keep the
      // register count high, and two CTAs per SM keep every token resident
      DG_CUDA(Launch(dim3(T), dim3(((d / 4 + 1) / 2 + 31) / 32 * 32), 0, st)(moe_combine_norm_kernel<2>, x, c->at<float>(L.yperm), c->at<int>(L.inv), T, k, d, g_next,
                                                 xn, m.rms_eps, pf, (long long)qkv_rows * d * 2));
      CNT(c);
    }
    DG_CUDA(cudaGetLastError());
    if (dbg_hidden)
      DG_CUDA(cudaMemcpyAsync(dbg_hidden + (size_t)(l + 1) * T * d, x, (size_t)T * d * 4,
                              cudaMemcpyDeviceToDevice, st));
  }
  return DG_OK;
}

static dg_status check_kv(const dg_ctx* c, const dg_kv* kv, int extra) {
  if (!kv || !kv->k || !kv->v) return fail(DG_ERR_INVALID_ARG, "kv buffers are null");
  if (kv->batch < 1 || kv->batch > c->batch_max) return fail(DG_ERR_INVALID_ARG, "kv batch %d outside [1, %d]", kv->batch, c->batch_max);
  if (kv->c_max < 8 || kv->c_max % 8) return fail(DG_ERR_INVALID_ARG, "kv c_max %d is not a positive multiple of 8", kv->c_max);
  if (kv->length < 0 || (long long)kv->length + extra > kv->c_max)
    return fail(DG_ERR_INVALID_ARG, "kv length %d + %d exceeds c_max %d", kv->length, extra, kv->c_max);
  return DG_OK;
}


extern "C" dg_status dg_encode_context(dg_ctx* c, dg_kv* kv, const int32_t* d_tokens, int32_t n, void* stream) {
  if (!c) return fail(DG_ERR_INVALID_ARG, "null context");
  if (n < 0) return fail(DG_ERR_INVALID_ARG, "n < 0");
  DG_TRY(check_kv(c, kv, n));
  if (n == 0) return DG_OK;
  if (!d_tokens) return fail(DG_ERR_INVALID_ARG, "tokens are null");
  cudaStream_t st = (cudaStream_t)stream;
  NvtxRange nv("dg.encode_context");
  const int B = kv->batch, d = c->cfg.d_model;
  int* tok_tmp = c->at<int>(c->L.tok);  // [T] staging of the chunk's token ids
  // chunks of as many tokens per canvas as a layer pass of the workspace holds
  // (256, or more with a prefill workspace: one weight stream per chunk)
  const int chunk = std::max(DG_CANVAS, c->L.T_alloc / B / 8 * 8);
  for (int s0 = 0; s0 < n; s0 += chunk) {
    const int nq = std::min(chunk, n - s0);
    const int T = B * nq;
    // gather the chunk's tokens into a dense [B, nq] block
    DG_CUDA(cudaMemcpy2DAsync(tok_tmp, (size_t)nq * 4, d_tokens + s0, (size_t)n * 4, (size_t)nq * 4, B,
                              cudaMemcpyDeviceToDevice, st));
    DG_CUDA(Launch(dim3(T), dim3(128), 0, st)(embed_kernel, c->wp(c->wl.emb), tok_tmp, c->at<float>(c->L.x), T, d, c->cfg.vocab, c->err()));
    CNT(c);
    DG_CUDA(cudaGetLastError());
    DG_TRY(forward_layers(c, kv, B, nq, kv->length, nq, nullptr, nullptr, nullptr, nullptr, nullptr, st));
    kv->length += nq;
  }
  return DG_OK;
}

extern "C" dg_status dg_canvas_init(dg_ctx* c, dg_canvas* cv, int32_t block, uint64_t seed, void* stream) {
  if (!c || !cv || !cv->tokens || !cv->prev_argmax || !cv->done) return fail(DG_ERR_INVALID_ARG, "null canvas");
  if (cv->batch < 1 || cv->batch > c->batch_max) return fail(DG_ERR_INVALID_ARG, "canvas batch");
  if (block < 0 || block > (1 << 23)) return fail(DG_ERR_INVALID_ARG, "block index");
  cudaStream_t st = (cudaStream_t)stream;
  const int n = cv->batch * DG_CANVAS;
  canvas_init_kernel<<<(n + 255) / 256, 256, 0, st>>>(cv->tokens, cv->prev_argmax, cv->done, cv->locked, cv->batch, block,
                                                      (uint32_t)seed, (uint32_t)(seed >> 32), c->cfg.vocab);
                                                      CNT(c);
  DG_CUDA(cudaGetLastError());
  if (c->cfg.self_cond) {
    if (!cv->sc_state) return fail(DG_ERR_INVALID_ARG, "self-conditioning state is null");
    DG_CUDA(cudaMemsetAsync(cv->sc_state, 0, (size_t)n * c->cfg.d_model * 2, st));
  }
  return DG_OK;
}

static StepDev step_dev(const dg_step_args* a) {
  const dg_sampler_config& s = a->sampler;
  const double Ts = s.max_steps <= 1 ? (double)s.t_start
                                     : (double)s.t_start + ((double)s.t_end - (double)s.t_start) * a->step /
                                                               (double)(s.max_steps - 1);
  StepDev v;
  v.step = a->step;
  v.max_steps = s.max_steps;
  v.block = a->block;
  v.policy = s.lock_policy;
  v.lock_threshold = s.lock_threshold;
  v.stop_entropy = s.stop_entropy;
  v.inv_t = (float)(1.0 / Ts);
  v.require_stable = s.stop_require_stable_argmax;
  v.k0 = (uint32_t)s.seed;
  v.k1 = (uint32_t)(s.seed >> 32);
  v.persistent = s.persistent_lock != 0;
  return v;
}

static dg_status check_round_args(dg_ctx* c, const dg_kv* kv, dg_canvas* cv, const dg_step_args* a) {
  if (!c || !cv || !a) return fail(DG_ERR_INVALID_ARG, "null argument");
  DG_TRY(check_kv(c, kv, DG_CANVAS));
  if (cv->batch != kv->batch) return fail(DG_ERR_INVALID_ARG, "canvas batch %d != kv batch %d", cv->batch, kv->batch);
  if (!cv->tokens || !cv->prev_argmax || !cv->done || (c->cfg.self_cond && !cv->sc_state))
    return fail(DG_ERR_INVALID_ARG, "canvas buffers are null");
  const dg_sampler_config& s = a->sampler;
  if (s.max_steps < 1 || s.max_steps > 256 || a->step < 0 || a->step >= s.max_steps || a->block < 0 ||
      a->block > (1 << 23))
    return fail(DG_ERR_INVALID_ARG, "step %d / max_steps %d / block %d out of range", a->step, s.max_steps, a->block);
  if (s.lock_policy != DG_LOCK_PROB && s.lock_policy != DG_LOCK_ENTROPY_CUMSUM)
    return fail(DG_ERR_INVALID_ARG, "lock policy");
  if (!(s.t_start > 0.f) || !(s.t_end > 0.f)) return fail(DG_ERR_INVALID_ARG, "temperatures must be > 0");
  if (s.persistent_lock && !cv->locked) return fail(DG_ERR_INVALID_ARG, "persistent lock needs canvas.locked");
  if (s.selfcond_topk < 0 || s.selfcond_topk > std::min(kTopkMax, c->cfg.vocab))
    return fail(DG_ERR_INVALID_ARG, "selfcond_topk %d outside [0, %d]", s.selfcond_topk,
                std::min(kTopkMax, c->cfg.vocab));
  return DG_OK;
}

// Enqueue one round.  The first launch writes the round parameters to the
// device (its node is returned when the stream is being captured).  With
// `append` ([B, 256] tokens of a finished block), the block is appended to
// the context in the same pass: each canvas's pass holds 512 tokens, the
// block's (causal, positions L0 ..) then the canvas's (bidirectional,
// positions L0 + 256 ..); the vocabulary phase runs on the canvas rows only.
static dg_status enqueue_round(dg_ctx* c, const dg_kv* kv, dg_canvas* cv, const dg_step_args* a,
                               const dg_step_out* o, cudaStream_t st, cudaGraphNode_t* param_node,
                               const int32_t* append = nullptr) {
  const dg_model_config& m = c->cfg;
  const WsLayout& L = c->L;
  const dg_sampler_config& s = a->sampler;
  const int B = cv->batch, T = B * DG_CANVAS, d = m.d_model, V = m.vocab;
  int* err = c->err();
  const int bnT = token_bn(T);
  dg_step_out none{};
  if (!o) o = &none;
  StepDev* sp = c->at<StepDev>(L.stepdev);
  step_params_kernel<<<1, 32, 0, st>>>(sp, step_dev(a));
  CNT(c);
  DG_CUDA(cudaGetLastError());
  if (param_node) {
    cudaStreamCaptureStatus cs;
    const cudaGraphNode_t* deps = nullptr;
    size_t nd = 0;
    DG_CUDA(cudaStreamGetCaptureInfo(st, &cs, nullptr, nullptr, &deps, &nd));
    if (cs != cudaStreamCaptureStatusActive || nd != 1) return fail(DG_ERR_CUDA, "capture of the round failed");
    *param_node = deps[0];
  }

  // a1: canvas embedding (+ self-conditioning input)
  NvtxRange nv_round("dg.denoise_step");
  const int nq = append ? 2 * DG_CANVAS : DG_CANVAS;   // tokens per canvas in the pass
  if (append) {
    // the pass's token ids, [B][block | canvas]; the embedding of all of them
    int* tok = c->at<int>(L.tok);
    DG_CUDA(cudaMemcpy2DAsync(tok, (size_t)nq * 4, append, (size_t)DG_CANVAS * 4, (size_t)DG_CANVAS * 4, B,
                              cudaMemcpyDeviceToDevice, st));
    DG_CUDA(cudaMemcpy2DAsync(tok + DG_CANVAS, (size_t)nq * 4, cv->tokens, (size_t)DG_CANVAS * 4,
                              (size_t)DG_CANVAS * 4, B, cudaMemcpyDeviceToDevice, st));
    DG_CUDA(Launch(dim3(B * nq), dim3(128), 0, st)(embed_kernel, c->wp(c->wl.emb), tok, c->at<float>(L.x), B * nq, d, V, err));
    CNT(c);
    DG_CUDA(cudaGetLastError());
  }
  if (m.self_cond) {
    ProfScope ps_(c, DG_PROF_DENSE, st);
    CUtensorMap ta;
    BOperand tb;
    const int bn = dense_bn((d + 127) / 128, T, c->num_sms);
    DG_TRY(make_tmap(&ta, c->wp(c->wl.sc), d, d, 128));
    DG_TRY(make_bop(&tb, cv->sc_state, d, T, bn));
    GemmPlan p = dense_plan(d, d, T, bn, 1, err);
    p.a_hint = 1;
    EpiStoreT e{c->at<float>(L.x), d, 0, 2, c->wp(c->wl.emb), cv->tokens, V, err};
    if (append) {  // canvas token t goes to pass row (t / 256) * 512 + 256 + t % 256
      e.row_group = DG_CANVAS;
      e.row_pitch = nq;
      e.row_off = DG_CANVAS;
    }
    DG_TRY(run_gemm(ta, tb, p, e, c->num_sms, st, &c->n_launch));
  } else if (!append) {
    DG_CUDA(Launch(dim3(T), dim3(128), 0, st)(embed_kernel, c->wp(c->wl.emb), cv->tokens, c->at<float>(L.x), T, d, V, err));
    CNT(c);
    DG_CUDA(cudaGetLastError());
  }

  if (o->hidden)
    DG_CUDA(cudaMemcpyAsync(o->hidden, c->at<float>(L.x), (size_t)T * d * 4, cudaMemcpyDeviceToDevice, st));

  // a2-a6: transformer layers, bidirectional over the canvas (the appended
  // block's tokens causal)
  DG_TRY(forward_layers(c, kv, B, nq, kv->length, append ? DG_CANVAS : 0, o->route_idx, o->route_w,
                        o->route_logits, o->hidden, o->hidden_attn, st));
  if (append) {
    // the canvas rows of the final normed stream, compacted for the LM head
    const size_t row = (size_t)d * 2;
    DG_CUDA(cudaMemcpy2DAsync(c->at<uint16_t>(L.xnc), (size_t)DG_CANVAS * row, c->at<uint16_t>(L.xn) +
                              (size_t)DG_CANVAS * d, (size_t)nq * row, (size_t)DG_CANVAS * row, B,
                              cudaMemcpyDeviceToDevice, st));
  }

  // a7: final norm, LM head with online vocabulary statistics and sampling
  NvtxRange nv_lm("dg.vocabulary_phase");  // a7-a9: LM head, statistics, expected embedding, update
  // final RMSNorm: fused into the last layer's combine
  uint16_t* xn = append ? c->at<uint16_t>(L.xnc) : c->at<uint16_t>(L.xn);
  uint16_t* logits = c->at<uint16_t>(L.logits);  // bf16, the expected embedding's input
  VocabPartials vp{c->at<float>(L.vp_m), c->at<float>(L.vp_z), c->at<float>(L.vp_s), c->at<float>(L.vp_av),
                   c->at<int>(L.vp_ai), c->at<float>(L.vp_gv), c->at<int>(L.vp_gi)};
  {
    ProfScope ps_(c, DG_PROF_LM_HEAD, st);
    CUtensorMap ta;
    BOperand tb;
    // on CTA pairs: one tcgen05.mma.cta_group::2 covers 256 positions (both
    // CTAs' 128-row A tiles) x 256 vocabulary ids, each CTA copying 128 of
    // the ids; one CTA per SM (two 256-column accumulators per CTA)
    DG_TRY(make_tmap(&ta, xn, d, L.T_alloc, 128));
    DG_TRY(make_bop_half(&tb, c->wp(c->wl.lm), d, V, 256));
    GemmPlan p = dense_plan(d, T, V, 256, 1, err);
    p.n_fast = 0;
    p.a_hint = 2;
    p.b_hint = 1;
    EpiLMHead e{logits, o->logits, V, vp, L.n_vt, 256, sp, DG_CANVAS, kPurposeGumbel};
    DG_TRY(run_gemm_pair(ta, tb, p, e, c->num_sms, st, &c->n_launch));
  }
  PosStats ps{c->at<float>(L.st_m), c->at<float>(L.st_iz), o->entropy ? o->entropy : c->at<float>(L.st_h),
              o->pmax ? o->pmax : c->at<float>(L.st_pmax), o->argmax ? o->argmax : c->at<int>(L.st_amax),
              o->sample ? o->sample : c->at<int>(L.st_samp)};
  DG_CUDA(Launch(dim3(T), dim3(kMergeThreads), 0, st)(vocab_merge_kernel, vp.m, vp.z, vp.s, vp.amax_v, vp.amax_i, vp.gkey_v,
                                                  vp.gkey_i, L.n_vt, T, log((double)V), ps));
                                                           CNT(c);
  DG_CUDA(cudaGetLastError());

  // a8: expected embedding for the next round's self-conditioning input
  if (m.self_cond && s.selfcond_topk > 0) {
    // high-batch variant: over each position's K largest logits only
    NvtxRange nv_e("dg.expected_embedding");
    ProfScope ps_(c, DG_PROF_EXPECTED_EMB, st);
    DG_TRY(set_smem_attr((const void*)topk_esum_kernel, (int)sizeof(TopkSmem), false));
    DG_CUDA(Launch(dim3(std::min(T, c->num_sms)), dim3(kTopkThreads), sizeof(TopkSmem), st)(
        topk_esum_kernel, logits, (long long)V, s.selfcond_topk, c->wp(c->wl.emb), d, DG_CANVAS, T, cv->done,
        cv->sc_state));
    CNT(c);
    DG_CUDA(cudaGetLastError());
  } else if (m.self_cond) {
    NvtxRange nv_e("dg.expected_embedding");
    ProfScope ps_(c, DG_PROF_EXPECTED_EMB, st);
    uint16_t* probs = c->at<uint16_t>(L.probs);
    const long long n8 = (long long)T * V / 8;
    DG_CUDA(Launch(dim3((unsigned)std::min<long long>((n8 + 255) / 256, 148 * 16)), dim3(256), 0, st)(probs_kernel, logits, ps.m, ps.inv_z, probs, T, V));
        CNT(c);
    const int ks = esum_splits(m, T, c->num_sms);
    CUtensorMap ta;
    BOperand tb;
    DG_TRY(make_tmap(&ta, c->wp(c->wl.embT), V, d, 128));
    DG_TRY(make_bop(&tb, probs, V, L.T_canvas, bnT));
    GemmPlan p = dense_plan(V, d, T, bnT, ks, err);
    p.mt = kEsumMt;
    p.a_hint = 1;
    p.b_hint = 2;
    EpiStoreT e{c->at<float>(L.epart), d, (long long)T * d, 0, nullptr, nullptr, 0, err};
    DG_TRY(run_gemm(ta, tb, p, e, c->num_sms, st, &c->n_launch));
    const long long n = (long long)T * d;
    DG_CUDA(Launch(dim3((unsigned)std::min<long long>((n + 255) / 256, 148 * 16)), dim3(256), 0, st)(esum_kernel, c->at<float>(L.epart), ks, T, d, DG_CANVAS, cv->done, cv->sc_state));
        CNT(c);
    DG_CUDA(cudaGetLastError());
  }

  // a9: mean entropy, stop, lock, next canvas
  NvtxRange nv_u("dg.canvas_update");
  UpdateParams up{};
  up.entropy = ps.entropy;
  up.pmax = ps.pmax;
  up.argmax = ps.argmax;
  up.sample = ps.sample;
  up.tokens = cv->tokens;
  up.prev_argmax = cv->prev_argmax;
  up.done = cv->done;
  up.lock_out = o->lock;
  up.mean_out = o->mean_entropy;
  up.stop_out = o->stop;
  up.final_out = o->final_round;
  up.flags = c->at<uint8_t>(L.flags);
  up.locked = cv->locked;
  up.sp = sp;
  up.vocab = V;
  DG_CUDA(Launch(dim3(B), dim3(256), 0, st)(canvas_update_kernel, up));
  CNT(c);
  DG_CUDA(cudaGetLastError());
  return DG_OK;
}

extern "C" dg_status dg_denoise_step(dg_ctx* c, const dg_kv* kv, dg_canvas* cv, const dg_step_args* a,
                                     const dg_step_out* o, void* stream) {
  DG_TRY(check_round_args(c, kv, cv, a));
  return enqueue_round(c, kv, cv, a, o, (cudaStream_t)stream, nullptr);
}

extern "C" dg_status dg_denoise_step_append(dg_ctx* c, dg_kv* kv, dg_canvas* cv, const dg_step_args* a,
                                            const int32_t* d_append, const dg_step_out* o, void* stream) {
  DG_TRY(check_round_args(c, kv, cv, a));
  if (!d_append) return fail(DG_ERR_INVALID_ARG, "append tokens are null");
  DG_TRY(check_kv(c, kv, 2 * DG_CANVAS));
  if (c->L.T_alloc < 2 * cv->batch * DG_CANVAS)
    return fail(DG_ERR_WORKSPACE, "an appending round needs layer passes of %d tokens (dg_workspace_bytes_ex)",
                2 * cv->batch * DG_CANVAS);
  if (o && (o->hidden || o->hidden_attn))
    return fail(DG_ERR_INVALID_ARG, "an appending round has no hidden-state outputs");
  DG_TRY(enqueue_round(c, kv, cv, a, o, (cudaStream_t)stream, nullptr, d_append));
  kv->length += DG_CANVAS;
  return DG_OK;
}

static bool same_key(const dg_ctx::GraphKey& a, const dg_ctx::GraphKey& b) {
  const dg_kv &x = a.kv, &y = b.kv;
  const dg_canvas &p = a.cv, &q = b.cv;
  const dg_step_out &u = a.out, &w = b.out;
  return a.topk == b.topk && x.k == y.k && x.v == y.v && x.batch == y.batch && x.c_max == y.c_max &&
         x.length == y.length &&
         p.tokens == q.tokens && p.sc_state == q.sc_state && p.prev_argmax == q.prev_argmax && p.done == q.done &&
         p.batch == q.batch && p.locked == q.locked && u.argmax == w.argmax && u.sample == w.sample && u.entropy == w.entropy &&
         u.pmax == w.pmax && u.lock == w.lock && u.mean_entropy == w.mean_entropy && u.stop == w.stop &&
         u.final_round == w.final_round && u.logits == w.logits && u.route_idx == w.route_idx &&
         u.route_w == w.route_w && u.route_logits == w.route_logits && u.hidden == w.hidden &&
         u.hidden_attn == w.hidden_attn;
}

extern "C" dg_status dg_denoise_step_graph(dg_ctx* c, const dg_kv* kv, dg_canvas* cv, const dg_step_args* a,
                                           const dg_step_out* o, void* stream) {
  DG_TRY(check_round_args(c, kv, cv, a));
  if (c->prof) return enqueue_round(c, kv, cv, a, o, (cudaStream_t)stream, nullptr);
  dg_ctx::GraphKey key;
  memset(&key, 0, sizeof(key));
  key.kv = *kv;
  key.cv = *cv;
  if (o) key.out = *o;
  key.topk = a->sampler.selfcond_topk;
  if (!c->g_valid || !same_key(key, c->g_key)) {
    c->drop_graph();
    if (!c->g_stream) DG_CUDA(cudaStreamCreateWithFlags(&c->g_stream, cudaStreamNonBlocking));
    // make sure one-time attribute calls happen outside the capture
    DG_TRY(check_round_args(c, kv, cv, a));
    DG_CUDA(cudaStreamBeginCapture(c->g_stream, cudaStreamCaptureModeThreadLocal));
    cudaGraphNode_t node = nullptr;
    const long long n0 = c->n_launch;
    const dg_status r = enqueue_round(c, kv, cv, a, o, c->g_stream, &node);
    c->g_kernels = c->n_launch - n0;
    c->n_launch = n0;
    cudaGraph_t g = nullptr;
    const cudaError_t e = cudaStreamEndCapture(c->g_stream, &g);
    if (r != DG_OK) {
      if (g) cudaGraphDestroy(g);
      return r;
    }
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "cudaStreamEndCapture: %s", cudaGetErrorString(e));
    cudaGraphExec_t ex = nullptr;
    const cudaError_t e2 = cudaGraphInstantiate(&ex, g, 0);
    if (e2 != cudaSuccess) {
      cudaGraphDestroy(g);
      return fail(DG_ERR_CUDA, "cudaGraphInstantiate: %s", cudaGetErrorString(e2));
    }
    c->g_graph = g;
    c->g_exec = ex;
    c->g_param_node = node;
    c->g_key = key;
    c->g_valid = true;
  }
  // this round's parameters go into the captured parameter node
  StepDev v = step_dev(a);
  StepDev* sp = c->at<StepDev>(c->L.stepdev);
  void* args[2] = {(void*)&sp, (void*)&v};
  cudaKernelNodeParams kp{};
  kp.func = (void*)step_params_kernel;
  kp.gridDim = dim3(1);
  kp.blockDim = dim3(32);
  kp.sharedMemBytes = 0;
  kp.kernelParams = args;
  kp.extra = nullptr;
  DG_CUDA(cudaGraphExecKernelNodeSetParams(c->g_exec, c->g_param_node, &kp));
  DG_CUDA(cudaGraphLaunch(c->g_exec, (cudaStream_t)stream));
  c->n_launch += c->g_kernels;
  return DG_OK;
}

// Retained autoregressive mode: one token per canvas through the layers
// (causal, appended to the context), then the final norm, LM head and
// statistics of that position: argmax and the Gumbel-max draw of the next
// token at `temperature`.
extern "C" dg_status dg_ar_step(dg_ctx* c, dg_kv* kv, const int32_t* d_tokens, float temperature, uint64_t seed,
                                int32_t* d_argmax, int32_t* d_sample, float* d_logits, void* stream) {
  if (!c || !d_tokens || !d_argmax || !d_sample) return fail(DG_ERR_INVALID_ARG, "null argument");
  if (!(temperature > 0.f)) return fail(DG_ERR_INVALID_ARG, "temperature must be > 0");
  DG_TRY(check_kv(c, kv, 1));
  cudaStream_t st = (cudaStream_t)stream;
  NvtxRange nv("dg.ar_step");
  const dg_model_config& m = c->cfg;
  const WsLayout& L = c->L;
  const int B = kv->batch, d = m.d_model, V = m.vocab, pos = kv->length;
  int* err = c->err();
  // round parameters of the draw: key = seed, c2 = the position
  StepDev v{};
  v.step = pos;
  v.max_steps = 1;
  v.block = 0;
  v.inv_t = (float)(1.0 / (double)temperature);
  v.k0 = (uint32_t)seed;
  v.k1 = (uint32_t)(seed >> 32);
  StepDev* sp = c->at<StepDev>(L.stepdev);
  step_params_kernel<<<1, 32, 0, st>>>(sp, v);
  CNT(c);
  DG_CUDA(Launch(dim3(B), dim3(128), 0, st)(embed_kernel, c->wp(c->wl.emb), d_tokens, c->at<float>(L.x), B, d, V, err));
  CNT(c);
  DG_CUDA(cudaGetLastError());
  DG_TRY(forward_layers(c, kv, B, 1, pos, 1, nullptr, nullptr, nullptr, nullptr, nullptr, st));
  kv->length += 1;
  uint16_t* xn = c->at<uint16_t>(L.xn);  // the final RMSNorm ran with the last layer's combine
  VocabPartials vp{c->at<float>(L.vp_m), c->at<float>(L.vp_z), c->at<float>(L.vp_s), c->at<float>(L.vp_av),
                   c->at<int>(L.vp_ai), c->at<float>(L.vp_gv), c->at<int>(L.vp_gi)};
  {
    CUtensorMap ta;
    BOperand tb;
    DG_TRY(make_tmap(&ta, xn, d, L.T_alloc, 128));
    DG_TRY(make_bop_half(&tb, c->wp(c->wl.lm), d, V, 256));
    GemmPlan p = dense_plan(d, B, V, 256, 1, err);
    p.n_fast = 0;
    p.a_hint = 2;
    p.b_hint = 1;
    EpiLMHead e{c->at<uint16_t>(L.logits), d_logits, V, vp, L.n_vt, 256, sp, 1, kPurposeArGumbel};
    DG_TRY(run_gemm_pair(ta, tb, p, e, c->num_sms, st, &c->n_launch));
  }
  PosStats ps{c->at<float>(L.st_m), c->at<float>(L.st_iz), c->at<float>(L.st_h), c->at<float>(L.st_pmax), d_argmax,
              d_sample};
  DG_CUDA(Launch(dim3(B), dim3(kMergeThreads), 0, st)(vocab_merge_kernel, vp.m, vp.z, vp.s, vp.amax_v, vp.amax_i, vp.gkey_v, vp.gkey_i,
                                                  L.n_vt, B, log((double)V), ps));
  CNT(c);
  DG_CUDA(cudaGetLastError());
  return DG_OK;
}

extern "C" dg_status dg_check_device_error(dg_ctx* c, void* stream) {
  if (!c) return fail(DG_ERR_INVALID_ARG, "null context");
  DG_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  int e = 0;
  DG_CUDA(cudaMemcpy(&e, c->err(), sizeof(int), cudaMemcpyDeviceToHost));
  if (e) {
    DG_CUDA(cudaMemset(c->err(), 0, sizeof(int)));
    // a wait that ran out may have left the routing counters mid-count
    DG_CUDA(cudaMemset(c->ws + c->L.rbar, 0, 64));
    DG_CUDA(cudaMemset(c->ws + c->L.rfill, 0, (size_t)c->cfg.n_experts * 8));
    if (e == kDevErrBadToken) return fail(DG_ERR_BAD_TOKEN, "a token id outside [0, vocab) reached the device");
    if (e == kDevErrTimeout) return fail(DG_ERR_TIMEOUT, "a bounded device wait ran out");
    return fail(DG_ERR_CUDA, "device error word %d", e);
  }
  return DG_OK;
}

extern "C" dg_status dg_decode_block(dg_ctx* c, dg_kv* kv, dg_canvas* cv, const dg_step_args* a, int32_t* d_out,
                                     dg_block_stats* h_stats, void* stream) {
  return dg_decode_block_ex(c, kv, cv, a, nullptr, 0, d_out, h_stats, stream);
}

extern "C" dg_status dg_decode_block_ex(dg_ctx* c, dg_kv* kv, dg_canvas* cv, const dg_step_args* a,
                                        const int32_t* d_pending, int32_t flags, int32_t* d_out,
                                        dg_block_stats* h_stats, void* stream) {
  if (!c || !cv || !a || !d_out) return fail(DG_ERR_INVALID_ARG, "null argument");
  if (flags & ~DG_DECODE_DEFER_APPEND) return fail(DG_ERR_INVALID_ARG, "unknown decode flags %d", flags);
  if (d_pending && d_pending == d_out) return fail(DG_ERR_INVALID_ARG, "the pending block and the output alias");
  DG_TRY(check_kv(c, kv, d_pending ? 2 * DG_CANVAS : DG_CANVAS));
  cudaStream_t st = (cudaStream_t)stream;
  NvtxRange nv("dg.decode_block");
  const int B = cv->batch;
  DG_TRY(dg_canvas_init(c, cv, a->block, a->sampler.seed, stream));
  std::vector<uint8_t> done_flags(B, 0);
  std::vector<int32_t> steps(B, 0);
  int rounds = 0, counted = 0;
  int* dstat = c->at<int>(c->L.dstat);
  const size_t dstat_bytes = (size_t)c->cfg.n_layers * 4;
  DG_CUDA(cudaMemsetAsync(dstat, 0, dstat_bytes, st));
  for (int s = 0; s < a->sampler.max_steps; ++s) {
    dg_step_args sa = *a;
    sa.step = s;
    if (s == 0 && d_pending) {
      DG_TRY(dg_denoise_step_append(c, kv, cv, &sa, d_pending, nullptr, stream));
      DG_CUDA(cudaMemsetAsync(dstat, 0, dstat_bytes, st));  // its pass routed the block's tokens too
    } else {
      DG_TRY(dg_denoise_step_graph(c, kv, cv, &sa, nullptr, stream));
      ++counted;
    }
    ++rounds;
    for (int b = 0; b < B; ++b)
      if (!done_flags[b]) ++steps[b];
    DG_CUDA(cudaMemcpyAsync(done_flags.data(), c->at<uint8_t>(c->L.flags), B, cudaMemcpyDeviceToHost, st));
    DG_TRY(dg_check_device_error(c, stream));  // synchronises the stream
    bool all = true;
    for (int b = 0; b < B; ++b) all = all && done_flags[b];
    if (all) break;
  }
  std::vector<int32_t> dsum(c->cfg.n_layers, 0);
  if (h_stats && h_stats->distinct_experts) {
    DG_CUDA(cudaMemcpyAsync(dsum.data(), dstat, dstat_bytes, cudaMemcpyDeviceToHost, st));
    DG_CUDA(cudaStreamSynchronize(st));
  }
  DG_CUDA(cudaMemcpyAsync(d_out, cv->tokens, (size_t)B * DG_CANVAS * 4, cudaMemcpyDeviceToDevice, st));
  if (!(flags & DG_DECODE_DEFER_APPEND)) DG_TRY(dg_encode_context(c, kv, d_out, DG_CANVAS, stream));
  if (h_stats) {
    h_stats->rounds = rounds;
    h_stats->tokens_per_pass = rounds ? (float)(B * DG_CANVAS) / (float)rounds : 0.f;
    if (h_stats->steps_taken) memcpy(h_stats->steps_taken, steps.data(), B * sizeof(int32_t));
    if (h_stats->distinct_experts)
      for (int l = 0; l < c->cfg.n_layers; ++l)
        h_stats->distinct_experts[l] = counted ? (float)dsum[l] / (float)counted : 0.f;
  }
  return DG_OK;
}

// Router-load probe: the RMSNorm, router product and routing of one layer on
// caller-given hidden states (the residual stream [T, d] fp32), as the layer
// runs them in a round; writes each token's experts.
extern "C" dg_status dg_router_probe(dg_ctx* c, int32_t layer, const float* d_x, int32_t T, int32_t* d_idx,
                                     void* stream) {
  if (!c || !d_x || !d_idx) return fail(DG_ERR_INVALID_ARG, "null argument");
  const dg_model_config& m = c->cfg;
  if (layer < 0 || layer >= m.n_layers) return fail(DG_ERR_INVALID_ARG, "layer %d outside [0, %d)", layer, m.n_layers);
  if (T < 1 || T > c->L.T_alloc) return fail(DG_ERR_INVALID_ARG, "T %d outside [1, %d]", T, c->L.T_alloc);
  cudaStream_t st = (cudaStream_t)stream;
  const WsLayout& L = c->L;
  const LayerW& W = c->wl.layers[layer];
  const int d = m.d_model, E = m.n_experts, k = m.top_k;
  int* err = c->err();
  float* x = c->at<float>(L.x);
  uint16_t* xn = c->at<uint16_t>(L.xn);
  DG_CUDA(cudaMemcpyAsync(x, d_x, (size_t)T * d * 4, cudaMemcpyDeviceToDevice, st));
  DG_CUDA(Launch(dim3(T), dim3(row_launch(d).threads), 0, st)(residual_norm_kernel<1>, x, nullptr, 0, 0, d, c->wp(W.g_moe), xn, m.rms_eps));
  DG_CUDA(cudaGetLastError());
  {
    CUtensorMap ta;
    BOperand tb;
    const int bn = std::max(32, dense_bn((E + 127) / 128, T, c->num_sms / L.ks_r));
    DG_TRY(make_tmap(&ta, c->wp(W.wr), d, c->wl.wr_rows, 128));
    DG_TRY(make_bop(&tb, xn, d, L.T_alloc, bn));
    GemmPlan p = dense_plan(d, E, T, bn, L.ks_r, err);
    if (DG_ROUTER_CLUSTER) p.cluster_k = L.ks_r;
    EpiStoreT e{c->at<float>(L.rpart), E, DG_ROUTER_CLUSTER ? 0 : (long long)T * E, 0, nullptr, nullptr, 0, err};
    DG_TRY(run_gemm(ta, tb, p, e, c->num_sms, st, &c->n_launch));
  }
  RouteParams rp;
  rp.part = c->at<float>(L.rpart);
  rp.xn = xn;
  rp.T = T; rp.E = E; rp.k = k; rp.d = d; rp.bn = 128;
  rp.tpc = (T + c->num_sms - 1) / c->num_sms;
  rp.off = c->at<int>(L.off);
  rp.chunk_off = c->at<int>(L.choff);
  rp.perm = c->at<int>(L.perm);
  rp.inv = c->at<int>(L.inv);
  rp.w_perm = c->at<float>(L.wperm);
  rp.xperm = c->at<uint16_t>(L.xperm);
  rp.fill = c->at<int>(L.rfill);
  rp.bar = c->at<int>(L.rbar);
  rp.dbg_idx = d_idx;
  rp.dbg_w = nullptr;
  rp.dbg_logits = nullptr;
  rp.dbg_nq = rp.dbg_skip = 0;
  rp.distinct = nullptr;
  rp.dep = nullptr;
  rp.dep_n = 0;
  rp.err = err;
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  lc.gridDim = dim3((T + rp.tpc - 1) / rp.tpc);
  lc.blockDim = dim3(kRouteThreads);
  lc.dynamicSmemBytes = route_smem_bytes(rp.tpc, k, E);
  lc.stream = st;
  lc.attrs = at;
  lc.numAttrs = 1;
  const int ksr = DG_ROUTER_CLUSTER ? 1 : L.ks_r;
  if (ksr == 8)      DG_CUDA(cudaLaunchKernelEx(&lc, route_kernel<8>, rp));
  else if (ksr == 4) DG_CUDA(cudaLaunchKernelEx(&lc, route_kernel<4>, rp));
  else if (ksr == 1) DG_CUDA(cudaLaunchKernelEx(&lc, route_kernel<1>, rp));
  else return fail(DG_ERR_UNSUPPORTED, "router split count %d", ksr);
  return DG_OK;
}

extern "C" dg_status dg_profile_start(dg_ctx* c) {
  if (!c) return fail(DG_ERR_INVALID_ARG, "null context");
  c->prof = true;
  c->n_launch = 0;
  c->ev_used = 0;
  c->prof_recs.clear();
  return DG_OK;
}

extern "C" dg_status dg_profile_stop(dg_ctx* c, dg_profile* out) {
  if (!c || !out) return fail(DG_ERR_INVALID_ARG, "null argument");
  c->prof = false;
  memset(out, 0, sizeof(*out));
  for (const auto& r : c->prof_recs) {
    DG_CUDA(cudaEventSynchronize(c->ev_pool[r.second + 1]));
    float ms = 0.f;
    DG_CUDA(cudaEventElapsedTime(&ms, c->ev_pool[r.second], c->ev_pool[r.second + 1]));
    out->ms[r.first] += ms;
    out->launches[r.first] += 1;
  }
  out->launches_total = c->n_launch;
  c->prof_recs.clear();
  c->ev_used = 0;
  return DG_OK;
}

// ============================================================================
// test hooks
namespace {
struct EpiGroupedT {
  static constexpr int kEpiWarps = 8;
  float* out;
  int ld;
  struct State {};
  __device__ __forceinline__ void begin(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void end(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void chunk(const GemmJob& j, int row, int c0, const float (&v)[16], State&) const {
    if (row >= j.m_valid) return;
    const int f = j.m_tile * 128 + row;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (c0 + i < j.n_valid) out[(long long)(j.n0 + c0 + i) * ld + f] = v[i];
  }
};

// row-major store; k split s writes the matrix at D + s * M * N
struct EpiSplitRows {
  static constexpr int kEpiWarps = 8;
  float* out;
  long long M, N;
  struct State {};
  __device__ __forceinline__ void begin(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void end(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void chunk(const GemmJob& j, int row, int c0, const float (&v)[16], State&) const {
    if (row >= j.m_valid) return;
    const long long m = (long long)j.m_tile * 128 + row;
    float* o = out + (long long)j.ks * M * N + m * N + j.n0;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (c0 + i < j.n_valid) o[c0 + i] = v[i];
  }
};
}  // namespace

extern "C" dg_status dg_test_gemm(const uint16_t* A, int32_t M, const uint16_t* B, int32_t N, int32_t K, float* D,
                                  int32_t k_splits, void* stream) {
  if (!A || !B || !D || M < 128 || N < 16 || K < 64 || K % 64 || k_splits < 1 || k_splits > K / 64)
    return fail(DG_ERR_INVALID_ARG, "dg_test_gemm: bad arguments");
  cudaStream_t st = (cudaStream_t)stream;
  int* err = nullptr;
  const int bn = token_bn(N);
  CUtensorMap ta;
  BOperand tb;
  DG_TRY(make_tmap(&ta, A, K, M, 128));
  DG_TRY(make_bop(&tb, B, K, N, bn));
  GemmPlan p = dense_plan(K, M, N, bn, k_splits, err);
  p.n_fast = 0;
  EpiSplitRows e{D, M, N};
  DG_TRY(run_gemm(ta, tb, p, e, device_sms(), st));
  DG_CUDA(cudaStreamSynchronize(st));
  return DG_OK;
}

extern "C" dg_status dg_test_gemm_tiles(const uint16_t* A, int32_t M, const uint16_t* B, int32_t N, int32_t K,
                                        float* D, int32_t k_splits, int32_t mt, int32_t bn, void* stream) {
  if (!A || !B || !D || M < 128 || N < 16 || K < 64 || K % 64 || k_splits < 1 || k_splits > K / 64 ||
      (mt != 1 && mt != 2) || (bn != 0 && (bn < 16 || bn > 256 || (bn & (bn - 1)))))
    return fail(DG_ERR_INVALID_ARG, "dg_test_gemm_tiles: bad arguments");
  cudaStream_t st = (cudaStream_t)stream;
  if (bn == 0) bn = token_bn(N);
  CUtensorMap ta;
  BOperand tb;
  DG_TRY(make_tmap(&ta, A, K, M, 128));
  DG_TRY(make_bop(&tb, B, K, N, bn));
  GemmPlan p = dense_plan(K, M, N, bn, k_splits, nullptr);
  p.n_fast = 0;
  p.mt = mt;
  EpiSplitRows e{D, M, N};
  DG_TRY(run_gemm(ta, tb, p, e, device_sms(), st));
  DG_CUDA(cudaStreamSynchronize(st));
  return DG_OK;
}

extern "C" dg_status dg_test_grouped_gemm(const uint16_t* A, int32_t rows_per_group, int32_t n_groups,
                                          const uint16_t* B, int32_t n_rows, int32_t K, const int32_t* off,
                                          float* D, int32_t bn, int32_t* choff, void* stream) {
  if (!A || !B || !D || !off || !choff || rows_per_group < 1 || n_groups < 1 || n_rows < 16 || K < 64 || K % 64 ||
      bn < 16 || bn > 256 || (bn & (bn - 1)))
    return fail(DG_ERR_INVALID_ARG, "dg_test_grouped_gemm: bad arguments");
  if ((long long)rows_per_group * n_groups < 128) return fail(DG_ERR_INVALID_ARG, "A needs >= 128 rows");
  cudaStream_t st = (cudaStream_t)stream;
  CUtensorMap ta;
  BOperand tb;
  DG_TRY(make_tmap(&ta, A, K, (long long)rows_per_group * n_groups, 128));
  DG_TRY(make_bop(&tb, B, K, n_rows, bn));
  chunk_offsets_kernel<<<1, 1, 0, st>>>(off, n_groups, bn, choff);
  GemmPlan p = grouped_plan(K, rows_per_group, off, choff, n_groups, bn, nullptr);
  EpiGroupedT e{D, rows_per_group};
  if (bn <= 128) {  // as in the layers: CTA pairs up to 128 rows per chunk
    BOperand th;
    DG_TRY(make_bop_half(&th, B, K, n_rows, bn));
    DG_TRY(run_gemm_pair(ta, th, p, e, device_sms(), st));
  } else {
    DG_TRY(run_gemm(ta, tb, p, e, device_sms(), st));
  }
  DG_CUDA(cudaStreamSynchronize(st));
  return DG_OK;
}

extern "C" dg_status dg_test_grouped_schedule(int32_t pair, int32_t rows_per_group, int32_t n_groups,
                                              const int32_t* off, int32_t K, int32_t bn, int32_t* jobs,
                                              int32_t max_jobs, int32_t* n_jobs) {
  if (!off || !n_jobs || (!jobs && max_jobs > 0) || max_jobs < 0 || rows_per_group < 1 || n_groups < 1 ||
      n_groups > kGemmMaxGroups || K < 64 || K % 64 || bn < 16 || bn > (pair ? 128 : 256) || (bn & (bn - 1)))
    return fail(DG_ERR_INVALID_ARG, "dg_test_grouped_schedule: bad arguments");
  GemmTables tb;
  tb.chunk_off[0] = 0;
  for (int g = 0; g <= n_groups; ++g) {
    tb.group_off[g] = off[g];
    if (g < n_groups) {
      const int rows = off[g + 1] - off[g];
      if (rows < 0) return fail(DG_ERR_INVALID_ARG, "dg_test_grouped_schedule: offsets decrease at %d", g);
      tb.chunk_off[g + 1] = tb.chunk_off[g] + (rows + bn - 1) / bn;
    }
  }
  GemmPlan p = grouped_plan(K, rows_per_group, off, tb.chunk_off, n_groups, bn, nullptr);
  const int rows[3] = {pair ? 8 : 16, pair ? std::min(32, bn / 2) : std::min(64, bn), pair ? bn / 2 : bn};
  for (int i = 0; i < 3; ++i) p.b_rows[i] = rows[i];
  const int U = pair ? pair_num_units(p, tb) : gemm_num_units(p, tb);
  const int ranks = pair ? 2 : 1;
  int n = 0;
  for (int u = 0; u < U; ++u)
    for (int r = 0; r < ranks; ++r, ++n) {
      if (n >= max_jobs) continue;
      const GemmJob j = pair ? pair_job(p, tb, u, r) : gemm_job(p, tb, u, 0);
      int32_t* o = jobs + (size_t)n * 10;
      o[0] = u; o[1] = r; o[2] = j.group; o[3] = j.m_tile; o[4] = j.a_row0; o[5] = j.m_valid;
      o[6] = j.n0; o[7] = j.n_valid; o[8] = j.kb1 - j.kb0; o[9] = pair ? pair_b_map(p, j.n_valid) : -1;
    }
  *n_jobs = n;
  return DG_OK;
}

extern "C" dg_status dg_test_dense_schedule(int32_t M, int32_t N, int32_t K, int32_t bn, int32_t k_splits,
                                           int32_t mt, int32_t n_fast, int32_t* jobs, int32_t max_jobs,
                                           int32_t* n_jobs) {
  if (!n_jobs || (!jobs && max_jobs > 0) || max_jobs < 0 || M < 1 || N < 1 || K < 64 || K % 64 || bn < 16 ||
      bn > 256 || (bn & (bn - 1)) || k_splits < 1 || k_splits > K / 64 || (mt != 1 && mt != 2))
    return fail(DG_ERR_INVALID_ARG, "dg_test_dense_schedule: bad arguments");
  GemmTables tb{};
  GemmPlan p = dense_plan(K, M, N, bn, k_splits, nullptr);
  p.mt = mt;
  p.n_fast = n_fast != 0;
  const int U = gemm_num_units(p, tb);
  int n = 0;
  for (int u = 0; u < U; ++u, ++n) {
    if (n >= max_jobs) continue;
    const GemmJob j = gemm_job(p, tb, u, 0);
    int32_t* o = jobs + (size_t)n * 8;
    o[0] = u; o[1] = j.m_tile; o[2] = j.mt_eff; o[3] = j.m_valid; o[4] = j.n0; o[5] = j.n_valid;
    o[6] = j.kb0; o[7] = j.kb1;
  }
  *n_jobs = n;
  return DG_OK;
}

extern "C" dg_status dg_test_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                                       int32_t B, int32_t nq, int32_t L0, int32_t c_max, int32_t Hq, int32_t Hkv,
                                       int32_t hd, int32_t causal, int32_t splits, float* part_o, float* part_ml,
                                       void* stream) {
  if (!q || !k || !v || !out || B < 1 || nq < 1 || L0 < 0 || L0 + nq > c_max || Hq < 1 || Hkv < 1 ||
      Hq % Hkv || splits < 0 || splits > kMaxAttnSplits)
    return fail(DG_ERR_INVALID_ARG, "dg_test_attention: bad arguments");
  cudaStream_t st = (cudaStream_t)stream;
  if (splits == 0) splits = 1;
  // no partial buffers: the splits merge inside their cluster
  const bool cluster = part_o == nullptr && part_ml == nullptr;
  if (causal < 0 || causal > nq) return fail(DG_ERR_INVALID_ARG, "dg_test_attention: causal %d", causal);
  DG_TRY(run_attention(q, k, v, out, part_o, part_ml, B, nq, L0, c_max, Hq, Hkv, hd, causal == 1 ? nq : causal,
                       splits, cluster, nullptr, st, nullptr));
  DG_CUDA(cudaStreamSynchronize(st));
  return DG_OK;
}

// One thread waits, with a bounded wait of limit_ns, on an mbarrier that
// nothing arrives on: the wait runs out, sets the error word and returns.
__global__ void wait_timeout_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(smem_u32(&bar), 1);
  fence_mbar_init();
  mbar_wait(smem_u32(&bar), 0, err, limit_ns);
}

extern "C" dg_status dg_test_wait_timeout(dg_ctx* c, int64_t limit_ns, void* stream) {
  if (!c || limit_ns <= 0 || limit_ns > 5000000000ll)
    return fail(DG_ERR_INVALID_ARG, "dg_test_wait_timeout: limit must be in (0, 5 s]");
  wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(c->err(), (unsigned long long)limit_ns);
  DG_CUDA(cudaGetLastError());
  return DG_OK;
}

extern "C" dg_status dg_test_expected_embedding_topk(const uint16_t* d_logits, int64_t V, int32_t K,
                                                     const uint16_t* d_emb, int32_t d, int32_t T, uint16_t* d_out,
                                                     void* stream) {
  if (!d_logits || !d_emb || !d_out || V < 256 || V % 256 || K < 1 || K > std::min<int64_t>(kTopkMax, V) ||
      d < 64 || d % 64 || d > 4096 || T < 1)
    return fail(DG_ERR_INVALID_ARG, "dg_test_expected_embedding_topk: bad arguments");
  cudaStream_t st = (cudaStream_t)stream;
  DG_TRY(set_smem_attr((const void*)topk_esum_kernel, (int)sizeof(TopkSmem), false));
  DG_CUDA(Launch(dim3(std::min(T, device_sms())), dim3(kTopkThreads), sizeof(TopkSmem), st, false)(
      topk_esum_kernel, d_logits, (long long)V, K, d_emb, d, DG_CANVAS, T, (const uint8_t*)nullptr, d_out));
  DG_CUDA(cudaStreamSynchronize(st));
  return DG_OK;
}

extern "C" size_t dg_test_struct_size(const char* name) {
  if (!name) return 0;
  const struct { const char* n; size_t s; } tab[] = {
      {"dg_model_config", sizeof(dg_model_config)}, {"dg_sampler_config", sizeof(dg_sampler_config)},
      {"dg_kv", sizeof(dg_kv)}, {"dg_canvas", sizeof(dg_canvas)}, {"dg_step_args", sizeof(dg_step_args)},
      {"dg_step_out", sizeof(dg_step_out)}, {"dg_block_stats", sizeof(dg_block_stats)},
      {"dg_profile", sizeof(dg_profile)}};
  for (const auto& e : tab)
    if (strcmp(e.n, name) == 0) return e.s;
  return 0;
}

extern "C" dg_status dg_test_workspace_buffer(dg_ctx* c, const char* name, void** ptr, size_t* bytes) {
  if (!c || !name || !ptr || !bytes) return fail(DG_ERR_INVALID_ARG, "null argument");
  const WsLayout& L = c->L;
  struct Entry { const char* n; size_t off, next; };
  const Entry tab[] = {{"x", L.x, L.xn}, {"xn", L.xn, L.qkv ? L.qkv : L.q}, {"q", L.q, L.attn},
                       {"attn", L.attn, L.rpart}, {"rpart", L.rpart, L.rbar},
                       {"off", L.off, L.perm}, {"perm", L.perm, L.inv}, {"inv", L.inv, L.wperm},
                       {"wperm", L.wperm, L.xperm}, {"xperm", L.xperm, L.hperm}, {"hperm", L.hperm, L.yperm},
                       {"yperm", L.yperm, L.logits}, {"logits", L.logits, L.vp_m},
                       {"probs", L.probs, L.epart}};
  for (const Entry& e : tab)
    if (!strcmp(e.n, name)) {
      if (!e.off && strcmp(name, "x")) return fail(DG_ERR_INVALID_ARG, "buffer %s not allocated", name);
      *ptr = c->ws + e.off;
      *bytes = e.next - e.off;
      return DG_OK;
    }
  return fail(DG_ERR_INVALID_ARG, "unknown workspace buffer %s", name);
}

// ============================================================================
// attention whose split-KV partials live in a fixed array of this library
// (for callers that cannot allocate device memory)

static __device__ __align__(256) float g_attn_scratch[DG_ATTN_STATIC_SCRATCH_BYTES / sizeof(float)];

static float* attn_scratch_address() {
  static std::mutex mu;
  static float* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess) return nullptr;
    addr[dev] = (float*)p;
  }
  return addr[dev];
}

extern "C" dg_status dg_attention_static_scratch(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                                 uint16_t* out, int32_t B, int32_t nq, int32_t L0, int32_t c_max,
                                                 int32_t Hq, int32_t Hkv, int32_t hd, int32_t causal,
                                                 int32_t splits, void* stream) {
  if (!q || !k || !v || !out || B < 1 || nq < 1 || L0 < 0 || L0 + nq > c_max || Hq < 1 || Hkv < 1 ||
      Hq % Hkv || splits < 0 || splits > kMaxAttnSplits)
    return fail(DG_ERR_INVALID_ARG, "dg_attention_static_scratch: bad arguments");
  const int sp = splits == 0 ? 1 : splits;
  const size_t rows = (size_t)sp * B * Hq * nq;
  const size_t o_floats = align_up(rows * hd, 64);
  const size_t need = (o_floats + rows * 2) * sizeof(float);
  if (sp > 1 && need > DG_ATTN_STATIC_SCRATCH_BYTES)
    return fail(DG_ERR_INVALID_ARG,
                "dg_attention_static_scratch: %zu bytes of split partials exceed the %u-byte scratch array",
                need, (unsigned)DG_ATTN_STATIC_SCRATCH_BYTES);
  float* base = attn_scratch_address();
  if (!base) return fail(DG_ERR_CUDA, "cudaGetSymbolAddress of the attention scratch failed");
  return dg_test_attention(q, k, v, out, B, nq, L0, c_max, Hq, Hkv, hd, causal, sp, base, base + o_floats,
                           stream);
}
