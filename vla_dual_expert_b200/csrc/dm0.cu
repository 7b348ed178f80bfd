// C ABI of the DM0 dual-expert merged-attention path (declared in dm0.h):
// context and buffer ownership, weight repacking, TMA descriptors, and the
// launch schedules of the prefix pass, the merged layer and the Euler loop.
//
// Schedule (DM0.5 page, sections 5.1-5.3 and 6.5):
//   prefill  : rows_prep, then per VLM layer
//              QKV GEMM (+QK-norm, RoPE, KV-cache write) -> attention
//              -> O GEMM (+residual, next-norm operand) -> gate/up GEMM (+SwiGLU)
//              -> down GEMM (+residual, next-norm operand)
//   denoise  : one observation of the DM0-base shapes: the whole Euler loop as one
//              persistent kernel (denoise_persistent.cuh).  Otherwise
//              step_kernel(input of step 0), then per step 28 action layers of
//              the same five kernels (attention over [prefix cache; suffix])
//              and step_kernel(velocity, Euler update, input of the next step),
//              captured once per (B, P, steps) into a CUDA graph and replayed.
//   options  : the FP8 E4M3 VLM MLP (dm0_set_prefix_fp8: per-token operand
//              quantisation + the kind::f8f6f4 GEMM), and the time-modulated
//              action expert (time_mod: per-loop modulation tables, then the
//              per-layer kernels with feature biases, gates and per-step gains).
// Every kernel is launched with programmatic stream serialization, so each
// kernel's prologue (TMEM allocation, barrier set-up, weight-tile requests)
// overlaps the previous kernel's tail.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "dm0.h"
#include "attention.cuh"
#include "attention_tc.cuh"
#include "attention_bwd.cuh"
#include "denoise_persistent.cuh"
#include "elementwise.cuh"
#include "gemm.cuh"
#include "ptx.cuh"
#include "train.cuh"

using dm0::AttnArgs;
using dm0::GemmArgs;
using dm0::StepArgs;
typedef __nv_bfloat16 bf16;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

struct LayerW {
  bf16 *wqkv, *wo, *wgu, *wd;
  float *attn_norm, *q_norm, *k_norm, *mlp_norm;
};

struct TmapKey {
  const void* p;
  uint64_t rows, cols;
  uint32_t box;
  bool operator<(const TmapKey& o) const {
    return std::tie(p, rows, cols, box) < std::tie(o.p, o.rows, o.cols, o.box);
  }
};

constexpr int kGemmStages = 4;
constexpr int kPartSlots = 1024;   // split-KV partial-state slots (x 128 rows)
constexpr int kGemmTraceLaunches = 64;   // DM0_GEMM_TRACE rows (persistent GEMM launches, round robin)

}  // namespace

struct dm0_ctx {
  dm0_config cfg{};
  int device = 0;
  int num_sms = 148;
  bool use_pdl = true, use_graph = true;
  // single-observation Euler loop as one persistent kernel (DM0_NO_PERSIST=1 selects the graph of
  // per-layer kernels instead); DM0_PERSIST_SPLITS overrides its attention key splits per KV head
  bool use_persist = true;
  int persist_splits = 7;
  bool qkv_epi4 = true;              // DM0_QKV_EPI=8: the QKV epilogue on eight warps (measured equal)
  bool persist_fast_bar = true;    // release-reduction grid barrier arrival (DM0_PERSIST_FASTBAR=0: full fences)
  int raster_band_override = 0;     // DM0_RASTER_BAND=n: persistent-GEMM bands of n m-tiles
  int persist_resident = -1;   // -1: not checked yet
  // true when the previous operation this context queued on the stream was one of its own
  // kernels: only then may the next kernel overlap it (programmatic dependent launch).  The first
  // kernel of every API call follows foreign work (caller kernels, copies) and waits for it in
  // plain stream order.
  bool pdl_ok = false;
  std::string err;

  void* wbuf = nullptr;
  LayerW* lw[2] = {nullptr, nullptr};
  std::vector<LayerW> lw_store[2];
  bf16 *W_in = nullptr, *W_out = nullptr;
  float *b_in = nullptr, *final_norm = nullptr, *b_out = nullptr;
  bool weights_loaded = false;

  bf16 *kplane = nullptr, *vplane = nullptr;
  int kv_B = 0, kv_P = 0;

  // VLM side, Mp = max_batch * max_prefix rows
  float* h_v = nullptr;
  bf16 *xn_v = nullptr, *q_v = nullptr, *o_v = nullptr, *act_v = nullptr;
  float* ssq_v = nullptr;
  // action side, Ms = max_batch * chunk rows
  float* h_a = nullptr;
  bf16 *xn_a = nullptr, *q_a = nullptr, *o_a = nullptr, *act_a = nullptr, *k_s = nullptr, *v_s = nullptr;
  float *ssq_a = nullptr, *x = nullptr;
  // split-K / split-KV scratch
  float* acc = nullptr;
  size_t acc_elems = 0;
  int* gcount = nullptr;
  int* acount = nullptr;
  int acount_n = 0;
  float* part_o = nullptr;
  float2* part_ml = nullptr;
  float2* rope = nullptr;
  float2* rope_t = nullptr;   // the same table dimension-major: [head_dim / 2][max_pos]
  int rope_max_pos = 0;
  int* d_err = nullptr;
  // dm0_infer_host staging
  bf16* stage_prefix = nullptr;
  // persistent Euler loop: split-K sums, sums of squares, grid-barrier words, per-layer norm gains
  float *pacc_qkv = nullptr, *pacc_gu = nullptr, *pssq = nullptr;
  unsigned* psync = nullptr;   // [0] barrier, [1] abort, [2 + g] suffix K/V flags
  bf16* pkv_sfx = nullptr;      // [n_kv][2][64][128] suffix K/V tiles built by the helper CTAs
  unsigned long long* ptrace = nullptr;   // DM0_PERSIST_TRACE=1: phase timestamps of the persistent loop
  unsigned long long* gtrace = nullptr;   // DM0_GEMM_TRACE=1: [kGemmTraceLaunches][num_sms][16] GEMM marks
  unsigned long long* atrace = nullptr;   // DM0_ATTN_TRACE=1: suffix-attention block marks (last launch)
  int gtrace_next = 0;                     // next launch slot (round robin)
  int ptrace_steps = 0;
  // FP8 E4M3 prefix MLP (dm0_set_prefix_fp8): per VLM layer the gate/up (interleaved as the bf16
  // copy) and down weights as codes with per-output-channel scales, and the per-token operands
  struct F8Layer {
    uint8_t *wgu, *wd;
    float *sgu, *sd;
  };
  // time-modulated action expert (cfg.time_mod): time MLP and modulator weights, and the tables of
  // every Euler step's scales, shifts and gates and of the shifts projected through the weights
  bf16 *tm_W_ti = nullptr, *tm_W_to = nullptr, *tm_Wmod = nullptr;   // [Ha][Ha] x 2, [(6L + 2) Ha][Ha]
  float *tm_b_ti = nullptr, *tm_b_to = nullptr, *tm_bmod = nullptr;
  int tm_cap = 0;                                                    // steps the tables hold
  bf16 *tm_tau = nullptr, *tm_act = nullptr, *tm_beta = nullptr;     // [cap][Ha] x 2, [L][2][cap][Ha]
  float *tm_c = nullptr, *tm_mod = nullptr;                          // [cap][Ha], [cap][(6L + 2) Ha]
  float *tm_bqkv = nullptr, *tm_bgu = nullptr;                       // [L][cap][QR], [L][cap][2 Ia]
  // flow-matching training step (dm0_train_step): transposed action weights (valid while
  // train_wt_ok), the layer inputs, and per-layer scratch reused from layer to layer
  struct TrainW {
    bf16 *wqkv_t, *wo_t, *wgu_t, *wd_t;   // [Ha][QR], [HqD][Ha], [Ha][2Ia], [Ia][Ha]
  };
  std::vector<TrainW> tw;
  bool train_wt_ok = false;
  struct TrainBuf {
    float *hs, *xt, *u, *rho1, *rho2, *rhof, *rho_q, *rho_k;
    float *raw, *qr, *kr, *vs, *prob, *of, *lse, *tmp, *h1, *gu, *rf, *dv, *drf;
    float *dh, *dh_alt, *dact, *dr, *dof, *dqr, *dK, *dV, *dgu_w;
    bf16 *r1, *r2, *of_bf, *act, *dgu, *dqkv, *dy_bf, *tA, *tB;
    bf16 *q_bf, *k_bf, *v_bf;   // tensor-core attention operands: q [T][Hq D], suffix K / V [B][Hkv][S][D]
    int* count;
  } tb{};
  bool train_alloc = false;
  bool fp8_mlp = false;
  std::vector<F8Layer> f8;
  uint8_t *xq_v = nullptr, *aq_v = nullptr;   // [Mp][hidden_v], [Mp][inter_v] codes
  float *sxq_v = nullptr, *saq_v = nullptr;   // [Mp] scales
  float* act32_v = nullptr;                   // [Mp][inter_v] SwiGLU output in fp32

  cudaStream_t cap_stream = nullptr;
  struct Graph {
    cudaGraphExec_t exec;
    uint64_t kernels;
  };
  std::map<std::tuple<int, int, int>, Graph> graphs;
  uint64_t launches = 0;   // kernels this context has put on a stream (graph replays count their kernels)
  // event probe around the launches of selected kernel sites (dm0_probe)
  int probe_mask = 0;
  std::vector<cudaEvent_t> probe_ev;
  size_t probe_used = 0;
  struct ProbeRec {
    int site, e0, e1;
  };
  std::vector<ProbeRec> probe_recs;
  std::map<TmapKey, CUtensorMap> tmaps;
  std::vector<void*> allocs;
};

namespace {

dm0_status fail(dm0_ctx* c, dm0_status st, const std::string& msg) {
  if (c) c->err = msg;
  return st;
}

#define CK(call)                                                                              \
  do {                                                                                        \
    cudaError_t e_ = (call);                                                                  \
    if (e_ != cudaSuccess) return fail(c, DM0_ECUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

#define TRY(expr)                  \
  do {                             \
    dm0_status s_ = (expr);        \
    if (s_ != DM0_OK) return s_;   \
  } while (0)

template <typename T>
dm0_status dalloc(dm0_ctx* c, T** p, size_t elems) {
  void* v = nullptr;
  const size_t bytes = elems * sizeof(T) > 0 ? elems * sizeof(T) : 16;
  cudaError_t e = cudaMalloc(&v, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(c, DM0_ENOMEM, "cudaMalloc of " + std::to_string(bytes) + " bytes failed: " + cudaGetErrorString(e));
  }
  c->allocs.push_back(v);
  *p = static_cast<T*>(v);
  return DM0_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int qkv_rows(const dm0_config& g) { return (g.n_q + 2 * g.n_kv) * g.head_dim; }
int hidden_of(const dm0_config& g, int br) { return br == 0 ? g.hidden_v : g.hidden_a; }
int inter_of(const dm0_config& g, int br) { return br == 0 ? g.inter_v : g.inter_a; }

dm0_status get_tmap(dm0_ctx* c, CUtensorMap* out, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box) {
  const TmapKey key{ptr, rows, cols, box};
  auto it = c->tmaps.find(key);
  if (it != c->tmaps.end()) {
    *out = it->second;
    return DM0_OK;
  }
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(c, DM0_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0 || cols % 64 != 0)
    return fail(c, DM0_EINVAL, "TMA operand must be 16-byte aligned with a multiple of 64 columns");
  CUtensorMap m;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t boxd[2] = {64, box};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, boxd, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(c, DM0_ECUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(r) + ")");
  c->tmaps[key] = m;
  *out = m;
  return DM0_OK;
}

// 2-D map without swizzle (row-major boxes of box_cols x box_rows): fp32 (esize 4) or bf16 (esize 2);
// the persistent Euler loop's operand copies and split-K reduce-adds
dm0_status get_tmap_plain(dm0_ctx* c, CUtensorMap* out, const void* ptr, int esize, uint64_t rows, uint64_t cols,
                          uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(c, DM0_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0 || (cols * esize) % 16 != 0 || (box_cols * esize) % 16 != 0)
    return fail(c, DM0_EINVAL, "TMA operand must be 16-byte aligned with 16-byte rows");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esize};
  cuuint32_t boxd[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(out, esize == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(ptr), dims, strides, boxd, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(c, DM0_ECUDA, "cuTensorMapEncodeTiled (plain) failed (" + std::to_string(r) + ")");
  return DM0_OK;
}

// 2-D map of FP8 codes (one byte each) with 128-byte swizzle: boxes of one 128-byte row (128 codes of K)
// x box_rows rows, the operand layout of the FP8 GEMM (the same bytes per row as a bf16 k-block)
dm0_status get_tmap_u8(dm0_ctx* c, CUtensorMap* out, const void* ptr, uint64_t rows, uint64_t cols,
                       uint32_t box_rows) {
  const TmapKey key{ptr, rows, cols, box_rows | 0x80000000u};   // kept apart from bf16 maps of the same pointer
  auto it = c->tmaps.find(key);
  if (it != c->tmaps.end()) {
    *out = it->second;
    return DM0_OK;
  }
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(c, DM0_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0 || cols % 128 != 0)
    return fail(c, DM0_EINVAL, "FP8 TMA operand must be 16-byte aligned with a multiple of 128 columns");
  CUtensorMap m;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t boxd[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, boxd, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(c, DM0_ECUDA, "cuTensorMapEncodeTiled (u8) failed (" + std::to_string(r) + ")");
  c->tmaps[key] = m;
  *out = m;
  return DM0_OK;
}

template <typename... KArgs, typename... Args>
dm0_status launch(dm0_ctx* c, cudaStream_t s, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                  Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (c->use_pdl && c->pdl_ok) ? 1 : 0;
  CK(cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...));
  c->pdl_ok = true;
  ++c->launches;
  return DM0_OK;
}

// CUDA-event pair around the launches of a probed kernel site: begin returns the first
// event's index (or -1 when the site is not probed or the pool is full)
int probe_event(dm0_ctx* c, cudaStream_t s) {
  if (c->probe_used >= c->probe_ev.size()) {
    if (c->probe_ev.size() >= 16384) return -1;
    for (int i = 0; i < 256; ++i) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return -1;
      c->probe_ev.push_back(e);
    }
  }
  if (cudaEventRecord(c->probe_ev[c->probe_used], s) != cudaSuccess) return -1;
  c->pdl_ok = false;   // the next kernel follows an event record, not one of our kernels
  return static_cast<int>(c->probe_used++);
}
int probe_begin(dm0_ctx* c, cudaStream_t s, int site) {
  return (c->probe_mask >> site) & 1 ? probe_event(c, s) : -1;
}
void probe_end(dm0_ctx* c, cudaStream_t s, int site, int e0) {
  if (e0 < 0) return;
  const int e1 = probe_event(c, s);
  if (e1 >= 0) c->probe_recs.push_back({site, e0, e1});
}

// ---------------------------------------------------------------- GEMM dispatch
// Raster of the persistent GEMM: weights of up to 64 MB (every DM0-base projection, bf16 or E4M3)
// stay in the 126 MB L2 for the whole launch under their evict-last policy, so the tiles run
// n-fastest and each activation tile is read from DRAM once, by the CTAs of one wave; larger
// weight matrices keep the default 64-m-tile bands.  DM0_RASTER_BAND=n forces bands of n m-tiles.
// DM0_GEMM_TRACE=1: each persistent GEMM launch gets the next of kGemmTraceLaunches rows of marks
unsigned long long* next_gemm_trace(dm0_ctx* c) {
  if (!c->gtrace) return nullptr;
  const int slot = c->gtrace_next++ % kGemmTraceLaunches;
  return c->gtrace + static_cast<size_t>(slot) * c->num_sms * dm0::kGemmTraceSlots;
}

int raster_band(const dm0_ctx* c, size_t weight_bytes) {
  if (c->raster_band_override > 0) return c->raster_band_override;
  return weight_bytes <= (size_t(64) << 20) ? 1 : 0;
}

dm0_status run_gemm(dm0_ctx* c, cudaStream_t s, const bf16* act, int tokens, int K, const bf16* W, int wrows,
                    GemmArgs g, int force_swap = -1, int force_splits = 0) {
  if (tokens <= 0) return DM0_OK;
  if (K % 64 != 0 || wrows % 128 != 0)
    return fail(c, DM0_ESHAPE, "GEMM needs K % 64 == 0 and weight rows % 128 == 0");
  const bool swap = force_swap >= 0 ? force_swap != 0 : tokens <= 128;
  const int KB = K / 64;
  g.K = K;
  g.tokens = tokens;
  g.err = c->d_err;
  g.counters = c->gcount;
  CUtensorMap ta, tb;
  if (swap) {
    if (tokens > 128) return fail(c, DM0_ESHAPE, "swapped GEMM takes at most 128 tokens");
    const int BN = tokens <= 64 ? 64 : 128;
    const int tiles = wrows / 128;
    if (tiles > 1024) return fail(c, DM0_ESHAPE, "too many feature tiles");
    int splits = force_splits > 0 ? force_splits : (c->num_sms + tiles / 2) / tiles;
    splits = splits < 1 ? 1 : (splits > KB ? KB : splits);
    const int kbps = (KB + splits - 1) / splits;
    splits = (KB + kbps - 1) / kbps;
    g.M = wrows;
    g.N = tokens;
    g.swap = 1;
    g.kb_per_split = kbps;
    if (g.mode != dm0::kModeResid && g.mode != dm0::kModeStoreF32) {
      if (static_cast<size_t>(tokens) * wrows > c->acc_elems) return fail(c, DM0_ESHAPE, "split-K scratch too small");
      g.acc = c->acc;
      g.ld_acc = wrows;
    }
    TRY(get_tmap(c, &ta, W, wrows, K, 128));
    TRY(get_tmap(c, &tb, act, tokens, K, BN));
    const dim3 grid(tiles, 1, splits);
    if (BN == 64)
      return launch(c, s, dm0::gemm_tc_kernel<64, kGemmStages>, grid, dim3(dm0::kGemmThreads),
                    dm0::GemmSmem<64, kGemmStages>::kBytes, ta, tb, g);
    return launch(c, s, dm0::gemm_tc_kernel<128, kGemmStages>, grid, dim3(dm0::kGemmThreads),
                  dm0::GemmSmem<128, kGemmStages>::kBytes, ta, tb, g);
  }
  const int mt = (tokens + 127) / 128;
  int BN = (wrows % 256 == 0) ? 256 : 128;
  // narrower tiles when the grid would leave SMs idle, but only while the narrower tiling still fits
  // in one wave: a tile's k-loop is a chain of dependent MMAs whose time hardly depends on the tile
  // width, so a second, partial wave of narrow tiles costs more than idle SMs (M = 816: the O and
  // down projections take 128-wide tiles, 112 CTAs, instead of 224 64-wide ones); a 64-wide tile
  // only for column-independent epilogues
  const int min_bn = (g.mode == dm0::kModeResid || g.mode == dm0::kModeStoreF32) ? 64 : 128;
  while (BN > min_bn && mt * (wrows / BN) < c->num_sms && mt * (wrows / (BN / 2)) <= c->num_sms) BN /= 2;
  g.M = tokens;
  g.N = wrows;
  g.swap = 0;
  g.kb_per_split = KB;
  g.band_m = raster_band(c, static_cast<size_t>(wrows) * K * 2);
  g.trace = next_gemm_trace(c);
  TRY(get_tmap(c, &ta, act, tokens, K, 128));
  TRY(get_tmap(c, &tb, W, wrows, K, BN));
  // persistent: at most one CTA per SM walking the tiles
  const int ntiles = mt * (wrows / BN);
  const dim3 grid(std::min(ntiles, c->num_sms));
  // as many stages as fit in ~192 KB: more bytes in flight per SM for the narrower tiles
  if (BN == 256)
    return g.mode == dm0::kModeQKV && c->qkv_epi4
               ? launch(c, s, dm0::gemm_tc_persistent<256, 4, false, 4>, grid, dim3(dm0::PGemmWarps<4>::kThreads),
                        dm0::PGemmSmem<256, 4, 4>::kBytes, ta, tb, g)
               : launch(c, s, dm0::gemm_tc_persistent<256, 4>, grid, dim3(dm0::PGemmWarps<8>::kThreads),
                        dm0::PGemmSmem<256, 4>::kBytes, ta, tb, g);
  if (BN == 128)
    return g.mode == dm0::kModeQKV && c->qkv_epi4
               ? launch(c, s, dm0::gemm_tc_persistent<128, 6, false, 4>, grid, dim3(dm0::PGemmWarps<4>::kThreads),
                        dm0::PGemmSmem<128, 6, 4>::kBytes, ta, tb, g)
               : launch(c, s, dm0::gemm_tc_persistent<128, 6>, grid, dim3(dm0::PGemmWarps<8>::kThreads),
                        dm0::PGemmSmem<128, 6>::kBytes, ta, tb, g);
  return launch(c, s, dm0::gemm_tc_persistent<64, 8>, grid, dim3(dm0::PGemmWarps<8>::kThreads), dm0::PGemmSmem<64, 8>::kBytes,
                ta, tb, g);
}

// FP8 E4M3 GEMM: act [tokens][K] codes with per-token scales sa, W [wrows][K] codes with per-row scales
// sw; always the persistent normal-orientation kernel (rows past `tokens` of the last 128-row tile are
// zero-filled by TMA and their stores predicated off), tile width by the same one-wave rule as bf16
dm0_status run_gemm_e4m3(dm0_ctx* c, cudaStream_t s, const uint8_t* act, const float* sa, int tokens, int K,
                         const uint8_t* W, const float* sw, int wrows, GemmArgs g) {
  if (tokens <= 0) return DM0_OK;
  if (K % 128 != 0 || wrows % 128 != 0)
    return fail(c, DM0_ESHAPE, "FP8 GEMM needs K % 128 == 0 and weight rows % 128 == 0");
  g.K = K;
  g.tokens = tokens;
  g.err = c->d_err;
  g.counters = c->gcount;
  g.row_scale = sa;
  g.col_scale = sw;
  const int mt = (tokens + 127) / 128;
  int BN = (wrows % 256 == 0) ? 256 : 128;
  const int min_bn = (g.mode == dm0::kModeResid || g.mode == dm0::kModeStoreF32) ? 64 : 128;
  while (BN > min_bn && mt * (wrows / BN) < c->num_sms && mt * (wrows / (BN / 2)) <= c->num_sms) BN /= 2;
  g.M = tokens;
  g.N = wrows;
  g.swap = 0;
  g.kb_per_split = K / 128;
  g.band_m = raster_band(c, static_cast<size_t>(wrows) * K);
  g.trace = next_gemm_trace(c);
  CUtensorMap ta, tb;
  TRY(get_tmap_u8(c, &ta, act, tokens, K, 128));
  TRY(get_tmap_u8(c, &tb, W, wrows, K, BN));
  const int ntiles = mt * (wrows / BN);
  const dim3 grid(std::min(ntiles, c->num_sms));
  if (BN == 256)
    return launch(c, s, dm0::gemm_tc_persistent<256, 4, true>, grid, dim3(dm0::PGemmWarps<8>::kThreads),
                  dm0::PGemmSmem<256, 4>::kBytes, ta, tb, g);
  if (BN == 128)
    return launch(c, s, dm0::gemm_tc_persistent<128, 6, true>, grid, dim3(dm0::PGemmWarps<8>::kThreads),
                  dm0::PGemmSmem<128, 6>::kBytes, ta, tb, g);
  return launch(c, s, dm0::gemm_tc_persistent<64, 8, true>, grid, dim3(dm0::PGemmWarps<8>::kThreads),
                dm0::PGemmSmem<64, 8>::kBytes, ta, tb, g);
}

// per-row E4M3 codes and scales of a matrix [rows][cols] (bf16 or fp32), each row optionally scaled by
// gain[c] and its pending RMSNorm factor from ssq[row] first
// (ssq: `ssq_slots` partial sums per row, slot-major with stride `ssq_stride`, added in slot order)
template <typename T>
dm0_status quant_rows(dm0_ctx* c, cudaStream_t s, const T* x, int rows, int cols, uint8_t* q, float* scale,
                      const float* gain = nullptr, const float* ssq = nullptr, int ssq_slots = 1, int ssq_stride = 0) {
  if (rows <= 0) return DM0_OK;
  if (cols <= 0 || cols % 8 != 0) return fail(c, DM0_ESHAPE, "E4M3 row quantisation needs cols % 8 == 0");
  return launch(c, s, dm0::quant_rows_e4m3_kernel<T>, dim3(rows), dim3(256), 0, x, rows, cols, gain, ssq, ssq_slots,
                ssq_stride > 0 ? ssq_stride : rows, 1.0f / cols, c->cfg.rms_eps, q, scale);
}

// ---------------------------------------------------------------- attention dispatch
dm0_status run_attn(dm0_ctx* c, cudaStream_t s, const bf16* q, int seq_q, const bf16* ka, const bf16* va, int len_a,
                    const bf16* kb, const bf16* vb, int len_b, bf16* o, int B, int splits_req, int a_stable,
                    float* lse = nullptr) {
  const dm0_config& g = c->cfg;
  const int G = g.n_q / g.n_kv;
  const int tiles = (G * seq_q + 127) / 128;
  const int groups = B * g.n_kv;
  const int nblk = (len_a + len_b + 63) / 64;
  if (nblk == 0 || seq_q == 0) return DM0_OK;
  int splits = splits_req;
  if (splits <= 0) {
    const int ctas = groups * tiles;
    splits = ctas >= c->num_sms ? 1 : (2 * c->num_sms + ctas - 1) / ctas;
  }
  if (splits > nblk) splits = nblk;
  while (splits > 1 && groups * tiles * splits > kPartSlots) --splits;
  // the combine keeps (m, l) of every split and row in the kernel's shared memory
  const int smem_bytes = g.head_dim == 128 ? dm0::AttnSmem<128>::kBytes
                                           : (g.head_dim == 64 ? dm0::AttnSmem<64>::kBytes : dm0::AttnSmem<32>::kBytes);
  while (splits > 1 && splits * 128 * 8 > smem_bytes) --splits;
  const int bps = (nblk + splits - 1) / splits;
  splits = (nblk + bps - 1) / bps;
  if (splits > 1 && groups * tiles > c->acount_n) return fail(c, DM0_ESHAPE, "attention split counters too small");
  AttnArgs a{};
  a.q = q;
  a.seq_q = seq_q;
  a.ka = ka;
  a.va = va;
  a.len_a = len_a;
  a.kb = kb;
  a.vb = vb;
  a.len_b = len_b;
  a.o = o;
  a.n_q = g.n_q;
  a.n_kv = g.n_kv;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(g.head_dim)));
  a.blocks_per_split = bps;
  a.a_stable = a_stable;
  a.part_o = c->part_o;
  a.part_ml = c->part_ml;
  a.counters = c->acount;
  a.err = c->d_err;
  a.lse = lse;
  if (g.head_dim == 128) {
    // tcgen05 flash attention, K/V tiles of both segments by TMA; keys split in 64-key blocks
    const int fblk = (len_a + 63) / 64 + (len_b + 63) / 64;
    int fs = splits_req;
    if (fs <= 0) {   // fill the SMs once (two CTAs per SM for the prefix kernel, one for the deep suffix
                     // kernel), at most 4 splits: the combine reads every split's partial O
      const int ctas = groups * tiles;
      const int slots = (len_b == 0 || groups * tiles <= c->num_sms / 8 ? 2 : 1) * c->num_sms;
      fs = std::max(1, std::min(4, (slots + ctas / 2) / ctas));
    }
    fs = std::min(fs, fblk);
    while (fs > 1 && groups * tiles * fs > kPartSlots) --fs;
    while (fs > 1 && fs * 128 * 8 > static_cast<int>(dm0::FaSmem::kOffBar)) --fs;   // combine keeps (m, l) in smem
    int fbps = (fblk + fs - 1) / fs;
    fs = (fblk + fbps - 1) / fbps;
    if (fs > 1 && groups * tiles > c->acount_n) return fail(c, DM0_ESHAPE, "attention split counters too small");
    a.blocks_per_split = fbps;
    CUtensorMap tk, tv, tkb, tvb;
    TRY(get_tmap(c, &tk, ka, static_cast<uint64_t>(groups) * len_a, 128, dm0::FaSmem::kKeys));
    TRY(get_tmap(c, &tv, va, static_cast<uint64_t>(groups) * len_a, 128, dm0::FaSmem::kKeys));
    if (len_b > 0) {
      TRY(get_tmap(c, &tkb, kb, static_cast<uint64_t>(groups) * len_b, 128, dm0::FaSmem::kKeys));
      TRY(get_tmap(c, &tvb, vb, static_cast<uint64_t>(groups) * len_b, 128, dm0::FaSmem::kKeys));
    } else {
      tkb = tk;
      tvb = tv;
    }
    const dim3 grid(tiles, groups, fs);
    // prefix pass (K/V blocks shared by many CTAs through L2), and the suffix attention of small
    // batches: two CTAs per SM, small enough (113 KB, 24.5K registers) to share an SM with a
    // swapped GEMM CTA, so neighbouring kernels overlap under programmatic dependent launch
    if (len_b == 0 || groups * tiles * fs <= c->num_sms / 2)
      return launch(c, s, dm0::fa_tc_kernel<2, 1>, grid, dim3(dm0::kFaThreads), dm0::FaSmemT<2, 1>::kBytes, tk, tv,
                    tkb, tvb, a);
    // merged suffix attention: the cached prefix is read from DRAM once; deeper K/V prefetch and
    // two P buffers so the softmax runs ahead of the PV MMAs
    if (static_cast<size_t>(groups) * tiles * fs <= kPartSlots) a.trace = c->atrace;
    return launch(c, s, dm0::fa_tc_kernel<dm0::kFaDeepStages, 2>, grid, dim3(dm0::FaWarps<2>::kThreads),
                  dm0::FaSmemT<dm0::kFaDeepStages, 2>::kBytes, tk, tv, tkb, tvb, a);
  }
  const dim3 grid(tiles, groups, splits);
  switch (g.head_dim) {
    case 128:
      return launch(c, s, dm0::attn_kernel<128>, grid, dim3(dm0::kAttnThreads), dm0::AttnSmem<128>::kBytes, a);
    case 64:
      return launch(c, s, dm0::attn_kernel<64>, grid, dim3(dm0::kAttnThreads), dm0::AttnSmem<64>::kBytes, a);
    default:
      return launch(c, s, dm0::attn_kernel<32>, grid, dim3(dm0::kAttnThreads), dm0::AttnSmem<32>::kBytes, a);
  }
}

dm0_status rows_prep(dm0_ctx* c, cudaStream_t s, const void* in, int in_bf16, float* h, bf16* xn, const float* gain,
                     float* ssq, int n_slots, int M, int H) {
  return launch(c, s, dm0::rows_prep_kernel, dim3((M + 7) / 8), dim3(256), 0, in, in_bf16, h, xn, gain, ssq,
                n_slots, M, M, H);
}

GemmArgs base_args(dm0_ctx* c) {
  GemmArgs g{};
  const dm0_config& cf = c->cfg;
  g.eps = cf.rms_eps;
  g.n_q = cf.n_q;
  g.n_kv = cf.n_kv;
  g.head_dim = cf.head_dim;
  g.rope = c->rope;
  g.rope_t = c->rope_t;
  g.rope_ld = c->rope_max_pos;
  return g;
}

// Per-step pointers of the time-modulated action expert for one layer (all into the tables built by
// tmod_precompute): the QKV and gate/up feature biases (each norm's shift through the weights), the
// attention and MLP gates, the MLP norm's 1 + scale, and the next layer's attention 1 + scale.
struct ModPtrs {
  const float *qkv_bias, *gate_o, *scale_m, *gu_bias, *gate_d, *next_scale;
};

// QKV projection of one branch with QK-norm + RoPE; K/V to [B][n_kv][kv_seq][D]
dm0_status layer_qkv(dm0_ctx* c, cudaStream_t s, int br, int l, const bf16* xn, const float* ssq_in, int tokens,
                     int seq, int pos_offset, bf16* q_out, bf16* k_out, bf16* v_out, const ModPtrs* mod = nullptr) {
  const LayerW& w = c->lw[br][l];
  const int H = hidden_of(c->cfg, br);
  GemmArgs g = base_args(c);
  g.w_stable = 1;
  g.mode = dm0::kModeQKV;
  g.ssq_in = ssq_in;
  g.ssq_slots = H / 64;
  g.ssq_stride = tokens;
  g.inv_hidden = 1.0f / H;
  g.q_out = q_out;
  g.k_out = k_out;
  g.v_out = v_out;
  g.q_gain = w.q_norm;
  g.k_gain = w.k_norm;
  g.seq_len = seq;
  g.pos_offset = pos_offset;
  g.kv_seq = seq;
  if (mod) g.col_bias = mod->qkv_bias;
  const int site = br == 0 ? DM0_SITE_VLM_QKV : DM0_SITE_ACT_QKV;
  const int e0 = probe_begin(c, s, site);
  TRY(run_gemm(c, s, xn, tokens, H, w.wqkv, qkv_rows(c->cfg), g));
  probe_end(c, s, site, e0);
  return DM0_OK;
}

// O-proj (+residual) -> gate/up (+SwiGLU) -> down (+residual) of one branch
dm0_status layer_rest(dm0_ctx* c, cudaStream_t s, int br, int l, int tokens, float* h, bf16* xn, const bf16* o,
                      bf16* act, float* ssq_mlp, const float* next_gain, float* next_ssq,
                      const ModPtrs* mod = nullptr) {
  const dm0_config& cf = c->cfg;
  const LayerW& w = c->lw[br][l];
  const int H = hidden_of(cf, br), I = inter_of(cf, br);
  GemmArgs g = base_args(c);
  g.w_stable = 1;
  g.mode = dm0::kModeResid;
  g.h = h;
  g.H = H;
  g.xn = xn;
  g.gain_next = mod ? mod->scale_m : w.mlp_norm;
  g.col_gate = mod ? mod->gate_o : nullptr;
  g.ssq_out = ssq_mlp;
  g.ssq_stride = tokens;
  const int so = br == 0 ? DM0_SITE_VLM_O : DM0_SITE_ACT_O;
  int e0 = probe_begin(c, s, so);
  TRY(run_gemm(c, s, o, tokens, cf.n_q * cf.head_dim, w.wo, H, g));
  probe_end(c, s, so, e0);
  // FP8 prefix MLP: each GEMM's bf16 operand is quantised per token first (its probe site covers both)
  const bool f8 = br == 0 && c->fp8_mlp;
  // FP8: the gate/up operand is the normalised residual rms(h) * g in fp32, quantised per token (the
  // GEMM's epilogue then has no pending 1/rms to apply), and SwiGLU writes fp32 for the down operand
  GemmArgs u = base_args(c);
  u.w_stable = 1;
  u.mode = dm0::kModeSwiGLU;
  u.ssq_in = ssq_mlp;
  u.ssq_slots = H / 64;
  u.ssq_stride = tokens;
  u.inv_hidden = 1.0f / H;
  u.act = act;
  u.inter = I;
  u.col_bias = mod ? mod->gu_bias : nullptr;
  const int su = br == 0 ? DM0_SITE_VLM_GATEUP : DM0_SITE_ACT_GATEUP;
  e0 = probe_begin(c, s, su);
  if (f8) {
    TRY(quant_rows(c, s, static_cast<const float*>(h), tokens, H, c->xq_v, c->sxq_v, w.mlp_norm, ssq_mlp, H / 64,
                   tokens));
    u.ssq_in = nullptr;
    u.act = nullptr;
    u.act_f32 = c->act32_v;
    TRY(run_gemm_e4m3(c, s, c->xq_v, c->sxq_v, tokens, H, c->f8[l].wgu, c->f8[l].sgu, 2 * I, u));
  } else {
    TRY(run_gemm(c, s, xn, tokens, H, w.wgu, 2 * I, u));
  }
  probe_end(c, s, su, e0);
  GemmArgs d = base_args(c);
  d.w_stable = 1;
  d.mode = dm0::kModeResid;
  d.h = h;
  d.H = H;
  d.xn = next_gain ? xn : nullptr;
  d.gain_next = next_gain;
  d.ssq_out = next_gain ? next_ssq : nullptr;
  d.ssq_stride = tokens;
  d.col_gate = mod ? mod->gate_d : nullptr;
  const int sd = br == 0 ? DM0_SITE_VLM_DOWN : DM0_SITE_ACT_DOWN;
  e0 = probe_begin(c, s, sd);
  if (f8) {
    TRY(quant_rows(c, s, static_cast<const float*>(c->act32_v), tokens, I, c->aq_v, c->saq_v));
    TRY(run_gemm_e4m3(c, s, c->aq_v, c->saq_v, tokens, I, c->f8[l].wd, c->f8[l].sd, H, d));
  } else {
    TRY(run_gemm(c, s, act, tokens, I, w.wd, H, d));
  }
  probe_end(c, s, sd, e0);
  return DM0_OK;
}

dm0_status enqueue_prefill(dm0_ctx* c, cudaStream_t s, const void* prefix_emb, int B, int P) {
  const dm0_config& cf = c->cfg;
  c->pdl_ok = false;
  const int M = B * P, L = cf.layers, D = cf.head_dim;
  const size_t lstride = static_cast<size_t>(B) * cf.n_kv * P * D;
  // sums of squares of the pending norms: [H / 64 groups][M] for the attention norm, then the MLP norm
  float* ssq_attn = c->ssq_v;
  float* ssq_mlp = ssq_attn + static_cast<size_t>(cf.hidden_v / 64) * M;
  TRY(rows_prep(c, s, prefix_emb, 1, c->h_v, c->xn_v, c->lw[0][0].attn_norm, ssq_attn, cf.hidden_v / 64, M,
                cf.hidden_v));
  for (int l = 0; l < L; ++l) {
    bf16* kl = c->kplane + l * lstride;
    bf16* vl = c->vplane + l * lstride;
    TRY(layer_qkv(c, s, 0, l, c->xn_v, ssq_attn, M, P, 0, c->q_v, kl, vl));
    const int e0 = probe_begin(c, s, DM0_SITE_VLM_ATTN);
    TRY(run_attn(c, s, c->q_v, P, kl, vl, P, nullptr, nullptr, 0, c->o_v, B, 1, 0));
    probe_end(c, s, DM0_SITE_VLM_ATTN, e0);
    const bool more = l + 1 < L;
    TRY(layer_rest(c, s, 0, l, M, c->h_v, c->xn_v, c->o_v, c->act_v, ssq_mlp,
                   more ? c->lw[0][l + 1].attn_norm : nullptr, more ? ssq_attn : nullptr));
  }
  return DM0_OK;
}

// The time-modulated expert's step: the final norm of step k_out takes its 1 + scale and shift, the
// input of step k_in its first attention norm's 1 + scale, and no time embedding (null tables: DM0)
struct StepMod {
  const float *final_scale, *final_shift, *attn_scale0;
};

dm0_status step(dm0_ctx* c, cudaStream_t s, int B, int k_out, int k_in, int steps, float* vel,
                const StepMod* mod = nullptr) {
  const dm0_config& cf = c->cfg;
  StepArgs a{};
  a.x = c->x;
  a.h = c->h_a;
  a.h_ts = cf.hidden_a;
  a.h_fs = 1;
  a.xn = c->xn_a;
  a.ssq = c->ssq_a;   // the attention norm's [Ha / 64][tokens] block
  a.n_slots = cf.hidden_a / 64;
  a.tokens = B * cf.chunk;
  a.W_in = c->W_in;
  a.b_in = c->b_in;
  a.attn_norm0 = c->lw[1][0].attn_norm;
  a.final_norm = c->final_norm;
  a.W_out = c->W_out;
  a.b_out = c->b_out;
  a.Ha = cf.hidden_a;
  a.A = cf.action_dim;
  a.eps = cf.rms_eps;
  a.k_out = k_out;
  a.k_in = k_in;
  a.steps = steps;
  a.vel = vel;
  const float* shift = nullptr;
  if (mod) {
    a.final_norm = mod->final_scale;
    a.attn_norm0 = mod->attn_scale0;
    shift = mod->final_shift;
  }
  const int e0 = probe_begin(c, s, DM0_SITE_STEP);
  TRY(launch(c, s, dm0::step_kernel, dim3(B * cf.chunk), dim3(256), sizeof(float) * cf.hidden_a, a, shift));
  probe_end(c, s, DM0_SITE_STEP, e0);
  return DM0_OK;
}

// Tables of the time-modulated expert for `steps` Euler steps (t_k = 1 - k/K): c(t_k) through the time
// MLP, every norm's [1 + scale | shift | gate] (one GEMM over all layers' modulators), and each
// layer's two shifts projected through its QKV and gate/up weights (the biases of those GEMMs).  Each
// weight is read once per Euler loop, not once per step.
dm0_status tmod_tables(dm0_ctx* c, int steps) {
  if (steps <= c->tm_cap) return DM0_OK;
  const dm0_config& g = c->cfg;
  const size_t cap = std::max(steps, 16), Ha = g.hidden_a, L = g.layers, R = (6 * L + 2) * Ha;
  // a larger loop gets new tables; graphs captured earlier keep using (and own) the old ones
  TRY(dalloc(c, &c->tm_tau, cap * Ha));
  TRY(dalloc(c, &c->tm_act, cap * Ha));
  TRY(dalloc(c, &c->tm_c, cap * Ha));
  TRY(dalloc(c, &c->tm_mod, cap * R));
  TRY(dalloc(c, &c->tm_beta, L * 2 * cap * Ha));
  TRY(dalloc(c, &c->tm_bqkv, L * cap * qkv_rows(g)));
  TRY(dalloc(c, &c->tm_bgu, L * cap * 2 * g.inter_a));
  c->tm_cap = static_cast<int>(cap);
  return DM0_OK;
}

dm0_status tmod_precompute(dm0_ctx* c, cudaStream_t s, int steps) {
  const dm0_config& g = c->cfg;
  const int Ha = g.hidden_a, L = g.layers, R = (6 * L + 2) * Ha, QR = qkv_rows(g), GU = 2 * g.inter_a;
  TRY(tmod_tables(c, steps));
  GemmArgs f = base_args(c);
  f.mode = dm0::kModeStoreF32;
  f.w_stable = 1;
  TRY(launch(c, s, dm0::tmod_tau_kernel, dim3(steps), dim3(256), 0, c->tm_tau, steps, Ha));
  f.out_f32 = c->tm_c;
  TRY(run_gemm(c, s, c->tm_tau, steps, Ha, c->tm_W_ti, Ha, f, 0));
  TRY(launch(c, s, dm0::tmod_bias_silu_kernel, dim3(steps), dim3(256), 0, static_cast<const float*>(c->tm_c),
             static_cast<const float*>(c->tm_b_ti), Ha, c->tm_act));
  TRY(run_gemm(c, s, c->tm_act, steps, Ha, c->tm_W_to, Ha, f, 0));
  TRY(launch(c, s, dm0::tmod_bias_silu_kernel, dim3(steps), dim3(256), 0, static_cast<const float*>(c->tm_c),
             static_cast<const float*>(c->tm_b_to), Ha, c->tm_act));
  f.out_f32 = c->tm_mod;
  TRY(run_gemm(c, s, c->tm_act, steps, Ha, c->tm_Wmod, R, f, 0));
  TRY(launch(c, s, dm0::tmod_finish_kernel, dim3((R + 255) / 256, steps), dim3(256), 0, c->tm_mod,
             static_cast<const float*>(c->tm_bmod), steps, L, Ha, c->tm_beta));
  for (int l = 0; l < L; ++l) {
    const LayerW& w = c->lw[1][l];
    f.out_f32 = c->tm_bqkv + static_cast<size_t>(l) * steps * QR;
    TRY(run_gemm(c, s, c->tm_beta + (static_cast<size_t>(l) * 2 + 0) * steps * Ha, steps, Ha, w.wqkv, QR, f, 0));
    f.out_f32 = c->tm_bgu + static_cast<size_t>(l) * steps * GU;
    TRY(run_gemm(c, s, c->tm_beta + (static_cast<size_t>(l) * 2 + 1) * steps * Ha, steps, Ha, w.wgu, GU, f, 0));
  }
  return DM0_OK;
}

// Euler loop over the KV cache; x already holds x_1
dm0_status enqueue_denoise(dm0_ctx* c, cudaStream_t s, int steps, float* vel) {
  const dm0_config& cf = c->cfg;
  c->pdl_ok = false;
  const int B = c->kv_B, P = c->kv_P, S = cf.chunk, L = cf.layers, D = cf.head_dim;
  const int Ms = B * S;
  const size_t lstride = static_cast<size_t>(B) * cf.n_kv * P * D;
  const bool tm = cf.time_mod != 0;
  const size_t Ha = cf.hidden_a, R = (6 * static_cast<size_t>(L) + 2) * Ha;
  // time-modulated expert: step k's row of the modulation table, layer l's [scale|shift|gate] x 2 at 6 l Ha
  auto mrow = [&](int k) { return c->tm_mod + static_cast<size_t>(k) * R; };
  auto step_mod = [&](int k_out, int k_in) {
    StepMod m{};
    // a non-null shift selects the modulated step (no time embedding on the input); at the loop's
    // start no velocity is formed and step 0's final-norm row is only a placeholder
    m.final_scale = mrow(k_out >= 0 ? k_out : 0) + 6 * L * Ha;
    m.final_shift = m.final_scale + Ha;
    m.attn_scale0 = k_in >= 0 ? mrow(k_in) : c->lw[1][0].attn_norm;
    return m;
  };
  if (tm) TRY(tmod_precompute(c, s, steps));
  StepMod sm = tm ? step_mod(-1, 0) : StepMod{};
  TRY(step(c, s, B, -1, 0, steps, vel, tm ? &sm : nullptr));
  for (int k = 0; k < steps; ++k) {
    for (int l = 0; l < L; ++l) {
      const bf16* kl = c->kplane + l * lstride;
      const bf16* vl = c->vplane + l * lstride;
      float* ssq_attn = c->ssq_a;
      float* ssq_mlp = ssq_attn + static_cast<size_t>(cf.hidden_a / 64) * Ms;
      const bool more = l + 1 < L;
      ModPtrs mp{};
      if (tm) {
        const float* ml = mrow(k) + 6 * static_cast<size_t>(l) * Ha;
        mp.qkv_bias = c->tm_bqkv + (static_cast<size_t>(l) * steps + k) * qkv_rows(cf);
        mp.gate_o = ml + 2 * Ha;
        mp.scale_m = ml + 3 * Ha;
        mp.gu_bias = c->tm_bgu + (static_cast<size_t>(l) * steps + k) * 2 * cf.inter_a;
        mp.gate_d = ml + 5 * Ha;
        mp.next_scale = more ? ml + 6 * Ha : nullptr;
      }
      TRY(layer_qkv(c, s, 1, l, c->xn_a, ssq_attn, Ms, S, P, c->q_a, c->k_s, c->v_s, tm ? &mp : nullptr));
      const int e0 = probe_begin(c, s, DM0_SITE_ACT_ATTN);
      TRY(run_attn(c, s, c->q_a, S, kl, vl, P, c->k_s, c->v_s, S, c->o_a, B, 0, 1));
      probe_end(c, s, DM0_SITE_ACT_ATTN, e0);
      const float* next_gain = more ? (tm ? mp.next_scale : c->lw[1][l + 1].attn_norm) : nullptr;
      TRY(layer_rest(c, s, 1, l, Ms, c->h_a, c->xn_a, c->o_a, c->act_a, ssq_mlp, next_gain,
                     more ? ssq_attn : nullptr, tm ? &mp : nullptr));
    }
    sm = tm ? step_mod(k, k + 1 < steps ? k + 1 : -1) : StepMod{};
    TRY(step(c, s, B, k, k + 1 < steps ? k + 1 : -1, steps, vel, tm ? &sm : nullptr));
  }
  return DM0_OK;
}

// The persistent Euler loop covers one observation of the DM0-base shapes: head_dim 128, at most
// 64 suffix tokens and 128 attention rows per KV head, 128-row weight tiles, and per GEMM phase at
// most kPdBTiles pairs (and two weight tiles) per CTA under the kernel's split (dm0::pd_pairs).  Fills
// everything of `a` but the stream-time
// fields; false (with the reason) sends the loop to the per-layer kernels.
bool persist_plan(dm0_ctx* c, int steps, float* vel, dm0::PdArgs* a, std::string* why) {
  const dm0_config& g = c->cfg;
  auto no = [&](const char* m) {
    *why = m;
    return false;
  };
  if (!c->use_persist) return no("disabled");
  if (c->persist_resident < 0) {   // once per context: can one CTA of the kernel live on every SM?
    int per_sm = 0, coop = 0;
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, c->device);
    const cudaError_t oe =
        g.time_mod ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dm0::denoise_persistent_kernel<true>,
                                                                   dm0::kPdThreads, dm0::PdSmem::kBytes)
                   : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dm0::denoise_persistent_kernel<false>,
                                                                   dm0::kPdThreads, dm0::PdSmem::kBytes);
    if (oe != cudaSuccess) per_sm = 0;
    cudaGetLastError();
    c->persist_resident = (coop && per_sm >= 1) ? 1 : 0;
  }
  if (!c->persist_resident) return no("the persistent kernel cannot be resident on every SM");
  if (g.head_dim != 128) return no("head_dim != 128");
  const int B = c->kv_B, P = c->kv_P, T = B * g.chunk, G = g.n_q / g.n_kv;
  if (B != 1 || T > 61 || G * T > 112) return no("more than one observation");   // RoPE rows fit a P buffer
  if (T % 2) return no("odd token count");   // bulk copies of T (max, sum) pairs need 16-byte sizes
  if (g.hidden_a % 128 || qkv_rows(g) % 128 || g.inter_a % 64) return no("shapes do not tile by 128");
  const int nsm = c->num_sms;
  const int nblk = (P + 63) / 64 + 1;
  int splits = std::min({c->persist_splits, dm0::kPdMaxSplits, nblk, nsm / g.n_kv});
  if (splits < 1) return no("too few SMs");
  const int bps = (nblk + splits - 1) / splits;
  splits = (nblk + bps - 1) / bps;   // every split owns at least one block
  // per GEMM phase (QKV, O, gate/up, down): tiles, k-blocks, landing bytes per staged pair
  const long land_per[4] = {256L * T, 140L * splits * T + 128, 256L * T, 512L * T};
  const int geo[4][2] = {{qkv_rows(g) / 128, g.hidden_a / 64},
                         {g.hidden_a / 128, g.n_q * 2},
                         {g.inter_a / 64, g.hidden_a / 64},
                         {g.hidden_a / 128, g.inter_a / 64}};
  for (int ph = 0; ph < 4; ++ph) {
    int per = 0;   // the longest pair range of the kernel's split (dm0::pd_pairs)
    for (int cc = 0; cc < nsm; ++cc) {
      int q0, q1;
      dm0::pd_pairs(geo[ph][0], geo[ph][1], cc, nsm, q0, q1);
      per = std::max(per, q1 - q0);
    }
    if (per > dm0::kPdBTiles || per > geo[ph][1]) return no("GEMM ranges too long for the staging area");
    if (per * land_per[ph] > static_cast<long>(dm0::PdSmem::kLandG)) return no("operand copies exceed the landing area");
  }
  if (g.n_kv * splits > kPartSlots) return no("partial-state slots");
  if (g.n_kv * (splits + 1) > nsm) return no("too few SMs for the attention items and their helpers");
  *a = dm0::PdArgs{};
  a->L = g.layers;
  a->T = T;
  a->P = P;
  a->steps = steps;
  a->Ha = g.hidden_a;
  a->Ia = g.inter_a;
  a->n_q = g.n_q;
  a->n_kv = g.n_kv;
  a->QR = qkv_rows(g);
  a->eps = g.rms_eps;
  a->scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(g.head_dim)));
  a->splits = splits;
  a->bps = bps;
  {
    // the gains sit at one stride per layer in the weight buffer (see the weight layout in dm0_create)
    const LayerW* w = c->lw[1];
    const ptrdiff_t stride = g.layers > 1 ? w[1].attn_norm - w[0].attn_norm : 0;
    for (int l = 0; l < g.layers; ++l)
      if (w[l].attn_norm != w[0].attn_norm + l * stride || w[l].q_norm != w[0].q_norm + l * stride ||
          w[l].k_norm != w[0].k_norm + l * stride || w[l].mlp_norm != w[0].mlp_norm + l * stride)
        return no("layer gains not evenly strided");
    a->attn_norm0 = w[0].attn_norm;
    a->q_norm0 = w[0].q_norm;
    a->k_norm0 = w[0].k_norm;
    a->mlp_norm0 = w[0].mlp_norm;
    a->norm_stride = static_cast<int>(stride);
  }
  a->rope = c->rope;
  a->h = c->h_a;
  a->acc_qkv = c->pacc_qkv;
  a->acc_gu = c->pacc_gu;
  a->ssq = c->pssq;
  a->part_o = reinterpret_cast<bf16*>(c->part_o);   // bf16 partials in the fp32 slot area
  a->part_ml = c->part_ml;
  a->sync = c->psync;
  a->kv_sfx = c->pkv_sfx;
  a->err = c->d_err;
  a->trace = steps <= c->ptrace_steps ? c->ptrace : nullptr;
  StepArgs& st = a->step;
  st.x = c->x;
  st.h = c->h_a;
  st.h_ts = g.hidden_a;
  st.h_fs = 1;
  st.xn = nullptr;
  st.ssq = nullptr;
  st.n_slots = 0;
  st.tokens = T;
  st.W_in = c->W_in;
  st.b_in = c->b_in;
  st.attn_norm0 = nullptr;
  st.final_norm = c->final_norm;
  st.W_out = c->W_out;
  st.b_out = c->b_out;
  st.Ha = g.hidden_a;
  st.A = g.action_dim;
  st.eps = g.rms_eps;
  st.steps = steps;
  st.vel = vel;
  a->fast_bar = c->persist_fast_bar ? 1 : 0;
  if (g.time_mod) {   // the tables tmod_precompute fills before the launch
    a->tm_mod = c->tm_mod;
    a->tm_bqkv = c->tm_bqkv;
    a->tm_bgu = c->tm_bgu;
    a->tm_R = (6 * g.layers + 2) * g.hidden_a;
  }
  return true;
}

dm0_status enqueue_denoise_persistent(dm0_ctx* c, cudaStream_t s, const dm0::PdArgs& a) {
  const dm0_config& g = c->cfg;
  const uint64_t L = g.layers;
  CUtensorMap tq, to, tgu, td, tk, tv;
  TRY(get_tmap(c, &tq, c->lw[1][0].wqkv, L * qkv_rows(g), g.hidden_a, 128));
  TRY(get_tmap(c, &to, c->lw[1][0].wo, L * g.hidden_a, static_cast<uint64_t>(g.n_q) * g.head_dim, 128));
  TRY(get_tmap(c, &tgu, c->lw[1][0].wgu, L * 2 * g.inter_a, g.hidden_a, 128));
  TRY(get_tmap(c, &td, c->lw[1][0].wd, L * g.hidden_a, g.inter_a, 128));
  const uint64_t kv_rows = L * g.n_kv * static_cast<uint64_t>(a.P);
  TRY(get_tmap(c, &tk, c->kplane, kv_rows, 128, 64));
  TRY(get_tmap(c, &tv, c->vplane, kv_rows, 128, 64));
  const uint64_t T = a.T, QR = qkv_rows(g), GU = 2 * static_cast<uint64_t>(g.inter_a);
  CUtensorMap tacc_qkv, th, tacc_gu;   // split-K reduce-add destinations, [T][features] fp32
  TRY(get_tmap_plain(c, &tacc_qkv, c->pacc_qkv, 4, T, QR, 128, 64));
  TRY(get_tmap_plain(c, &th, c->h_a, 4, T, g.hidden_a, 128, 64));
  TRY(get_tmap_plain(c, &tacc_gu, c->pacc_gu, 4, T, GU, 128, 64));
  CUtensorMap th_ld, tgu_ld, tqkv_ld, tpo;   // operand copies: [T] rows of one 64- or 128-column block
  TRY(get_tmap_plain(c, &th_ld, c->h_a, 4, T, g.hidden_a, 64, a.T));
  TRY(get_tmap_plain(c, &tgu_ld, c->pacc_gu, 4, T, GU, 128, a.T));
  TRY(get_tmap_plain(c, &tqkv_ld, c->pacc_qkv, 4, T, QR, 128, a.T));
  CUtensorMap tml;
  {   // split-attention partials: O as [slot][128 rows][128 dims] bf16, (max, sum) as [slot][128 rows] 8-byte
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(c, DM0_ECUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t nslot = static_cast<cuuint64_t>(g.n_kv) * a.splits;
    cuuint64_t d3[3] = {128, 128, nslot};
    cuuint64_t s3[2] = {128 * 2, 128 * 128 * 2};
    cuuint32_t b3[3] = {64, static_cast<cuuint32_t>(a.T), static_cast<cuuint32_t>(a.splits)};
    cuuint32_t e3[3] = {1, 1, 1};
    CUresult r = enc(&tpo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, c->part_o, d3, s3, b3, e3, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(c, DM0_ECUDA, "cuTensorMapEncodeTiled (partial O) failed (" + std::to_string(r) + ")");
    cuuint64_t d2[2] = {128, nslot};
    cuuint64_t s2[1] = {128 * 8};
    cuuint32_t b2[2] = {static_cast<cuuint32_t>(a.T), static_cast<cuuint32_t>(a.splits)};
    cuuint32_t e2[2] = {1, 1};
    r = enc(&tml, CU_TENSOR_MAP_DATA_TYPE_INT64, 2, c->part_ml, d2, s2, b2, e2, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(c, DM0_ECUDA, "cuTensorMapEncodeTiled (partial max/sum) failed (" + std::to_string(r) + ")");
  }
  if (g.time_mod) TRY(tmod_precompute(c, s, a.steps));
  CK(cudaMemsetAsync(c->psync, 0, (2 + g.n_kv) * sizeof(unsigned), s));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c->num_sms);
  cfg.blockDim = dim3(dm0::kPdThreads);
  cfg.dynamicSmemBytes = dm0::PdSmem::kBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // grid barriers: every CTA must be resident
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int e0 = probe_begin(c, s, DM0_SITE_LOOP);
  const cudaError_t le =
      g.time_mod ? cudaLaunchKernelEx(&cfg, dm0::denoise_persistent_kernel<true>, tq, to, tgu, td, tk, tv, tacc_qkv, th,
                                      tacc_gu, th_ld, tgu_ld, tqkv_ld, tpo, tml, a)
                 : cudaLaunchKernelEx(&cfg, dm0::denoise_persistent_kernel<false>, tq, to, tgu, td, tk, tv, tacc_qkv,
                                      th, tacc_gu, th_ld, tgu_ld, tqkv_ld, tpo, tml, a);
  if (le == cudaErrorCooperativeLaunchTooLarge) {   // fewer SMs available than the device has: use the
    cudaGetLastError();                             // per-layer kernels from now on
    c->persist_resident = 0;
    return DM0_ESTATE;
  }
  CK(le);
  probe_end(c, s, DM0_SITE_LOOP, e0);
  c->launches += 1;
  c->pdl_ok = false;
  return DM0_OK;
}

// The CUDA graph of the per-layer Euler loop for the context's current (kv_B, kv_P) and `steps`,
// captured (not launched) on first use and cached
dm0_status denoise_graph(dm0_ctx* c, int steps, const dm0_ctx::Graph** out) {
  const auto key = std::make_tuple(c->kv_B, c->kv_P, steps);
  auto it = c->graphs.find(key);
  if (it == c->graphs.end()) {
    CK(cudaStreamBeginCapture(c->cap_stream, cudaStreamCaptureModeThreadLocal));
    const uint64_t l0 = c->launches;
    dm0_status st = enqueue_denoise(c, c->cap_stream, steps, nullptr);
    const uint64_t nk = c->launches - l0;
    c->launches = l0;
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamEndCapture(c->cap_stream, &graph);
    if (st != DM0_OK) {
      if (graph) cudaGraphDestroy(graph);
      return st;
    }
    if (e != cudaSuccess) return fail(c, DM0_ECUDA, std::string("graph capture: ") + cudaGetErrorString(e));
    cudaGraphExec_t exec = nullptr;
    e = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) return fail(c, DM0_ECUDA, std::string("graph instantiate: ") + cudaGetErrorString(e));
    it = c->graphs.emplace(key, dm0_ctx::Graph{exec, nk}).first;
  }
  *out = &it->second;
  return DM0_OK;
}

dm0_status denoise_from_x(dm0_ctx* c, cudaStream_t s, int steps, float* vel) {
  // the time-modulation tables are allocated outside any capture (an allocation may synchronise)
  if (c->cfg.time_mod) TRY(tmod_tables(c, steps));
  {
    dm0::PdArgs pa;
    std::string why;
    if (persist_plan(c, steps, vel, &pa, &why)) {
      const dm0_status st = enqueue_denoise_persistent(c, s, pa);
      if (!(st == DM0_ESTATE && c->persist_resident == 0)) return st;   // else fall through
    }
  }
  if (vel || !c->use_graph || c->probe_mask) return enqueue_denoise(c, s, steps, vel);
  const dm0_ctx::Graph* gr = nullptr;
  TRY(denoise_graph(c, steps, &gr));
  CK(cudaGraphLaunch(gr->exec, s));
  c->launches += gr->kernels;
  return DM0_OK;
}

bool cfg_ok(const dm0_config& g, std::string* why) {
  auto bad = [&](const char* m) {
    *why = m;
    return false;
  };
  if (g.layers < 1) return bad("layers must be >= 1");
  if (g.head_dim != 32 && g.head_dim != 64 && g.head_dim != 128) return bad("head_dim must be 32, 64 or 128");
  if (g.n_q < 1 || g.n_kv < 1 || g.n_q % g.n_kv != 0) return bad("n_q must be a positive multiple of n_kv");
  if (g.hidden_v % 128 || g.hidden_a % 128) return bad("hidden sizes must be multiples of 128");
  if (g.inter_v % 128 || g.inter_a % 128) return bad("intermediate sizes must be multiples of 128");
  if ((g.n_q * g.head_dim) % 128 || (g.n_kv * g.head_dim) % 32) return bad("head layout must tile by 128 columns");
  if (qkv_rows(g) % 128) return bad("(n_q + 2 n_kv) * head_dim must be a multiple of 128");
  if (g.action_dim < 1 || g.action_dim > 64) return bad("action_dim must be in [1, 64]");
  if (g.chunk < 1 || g.max_batch < 1 || g.max_prefix < 1) return bad("chunk, max_batch, max_prefix must be >= 1");
  if (g.max_prefix + g.chunk > 65536) return bad("max_prefix + chunk must be <= 65536");
  if (static_cast<long long>(g.max_batch) * g.chunk > 1 << 20) return bad("max_batch * chunk too large");
  if (!(g.rms_eps > 0.f) || !(g.rope_theta > 1.f)) return bad("rms_eps must be > 0 and rope_theta > 1");
  if (g.time_mod != 0 && g.time_mod != 1) return bad("time_mod must be 0 or 1");
  return true;
}

size_t layer_bytes(const dm0_config& g, int br) {
  const size_t H = hidden_of(g, br), I = inter_of(g, br), D = g.head_dim;
  const size_t qd = g.n_q * D, kvd = g.n_kv * D;
  return 4 * (H + D + D + H) + 2 * (qd * H + 2 * kvd * H + H * qd + 2 * I * H + H * I);
}

size_t blob_bytes(const dm0_config& g) {
  const size_t Ha = g.hidden_a, A = g.action_dim;
  size_t n = g.layers * (layer_bytes(g, 0) + layer_bytes(g, 1)) + 2 * Ha * A + 4 * Ha + 4 * Ha + 2 * A * Ha + 4 * A;
  // time MLP (2 x [Ha][Ha] + biases), final modulator ([2Ha][Ha] + bias), two [3Ha][Ha] modulators per layer
  if (g.time_mod) n += 8 * Ha * Ha + 16 * Ha + g.layers * (12 * Ha * Ha + 24 * Ha);
  return n;
}

}  // namespace

// ====================================================================== allocation-free attention
//
// Scratch for dm0_attention_noalloc: the split-KV partial states and arrival
// counters live in this file-scope device array instead of memory from
// cudaMalloc.  Every GPU that loads the library holds it (about 2 MB) until the
// process exits.  In host code the name is only a host-side stand-in; the
// device address is fetched per device with cudaGetSymbolAddress.
constexpr int kNoAllocSlots = 32;                               // (group x row tile x split) partial states
constexpr int kNoAllocOFloats = kNoAllocSlots * 128 * 128;      // partial O, head_dim up to 128
constexpr int kNoAllocMlFloats = kNoAllocSlots * 128 * 2;       // (m, l) per partial row
constexpr int kNoAllocCounters = kNoAllocSlots;                 // one arrival counter per (group, row tile)
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocOFloats + kNoAllocMlFloats + kNoAllocCounters];
// the split combine keeps (m, l) of every split of a row tile (128 rows x 8 bytes each) in the kernel's
// shared memory: the most splits the slots allow must fit the smallest instance
static_assert(kNoAllocSlots * 128 * 8 <= dm0::AttnSmem<32>::kBytes, "no-alloc splits exceed the combine's smem");

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_base[kNoAllocMaxDevices] = {};

// Once per device, with that device current: the array's device address and the
// attention kernels' shared-memory limit.
dm0_status noalloc_setup(int dev, float** base) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_base[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return DM0_ECUDA;
    if (cudaFuncSetAttribute(dm0::attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dm0::AttnSmem<128>::kBytes) != cudaSuccess ||
        cudaFuncSetAttribute(dm0::attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dm0::AttnSmem<64>::kBytes) != cudaSuccess ||
        cudaFuncSetAttribute(dm0::attn_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dm0::AttnSmem<32>::kBytes) != cudaSuccess)
      return DM0_ECUDA;
    g_noalloc_base[dev] = static_cast<float*>(p);
  }
  *base = g_noalloc_base[dev];
  return DM0_OK;
}
}  // namespace

// ====================================================================== C ABI

namespace {
// FP8 prefix MLP buffers, allocated on first use: per VLM layer the gate/up and down codes and scales,
// and the per-token operand codes and scales for max_batch * max_prefix tokens
dm0_status ensure_fp8(dm0_ctx* c) {
  if (!c->f8.empty()) return DM0_OK;
  const dm0_config& g = c->cfg;
  const size_t H = g.hidden_v, I = g.inter_v;
  const size_t Mp = static_cast<size_t>(g.max_batch) * g.max_prefix;
  std::vector<dm0_ctx::F8Layer> f8(g.layers);
  for (auto& w : f8) {
    TRY(dalloc(c, &w.wgu, 2 * I * H));
    TRY(dalloc(c, &w.sgu, 2 * I));
    TRY(dalloc(c, &w.wd, H * I));
    TRY(dalloc(c, &w.sd, H));
  }
  TRY(dalloc(c, &c->xq_v, Mp * H));
  TRY(dalloc(c, &c->aq_v, Mp * I));
  TRY(dalloc(c, &c->sxq_v, Mp));
  TRY(dalloc(c, &c->saq_v, Mp));
  TRY(dalloc(c, &c->act32_v, Mp * I));
  c->f8 = std::move(f8);
  return DM0_OK;
}

// codes and per-output-channel scales of every VLM layer's gate/up and down weights, from the bf16 copy
dm0_status pack_fp8_weights(dm0_ctx* c, cudaStream_t s) {
  const dm0_config& g = c->cfg;
  const int H = g.hidden_v, I = g.inter_v;
  c->pdl_ok = false;
  for (int l = 0; l < g.layers; ++l) {
    const LayerW& w = c->lw[0][l];
    TRY(quant_rows(c, s, w.wgu, 2 * I, H, c->f8[l].wgu, c->f8[l].sgu));
    TRY(quant_rows(c, s, w.wd, H, I, c->f8[l].wd, c->f8[l].sd));
  }
  return DM0_OK;
}
}  // namespace

#include "train_host.cuh"

extern "C" {

size_t dm0_weights_bytes(const dm0_config* cfg) { return cfg ? blob_bytes(*cfg) : 0; }

dm0_status dm0_create(const dm0_config* cfg, dm0_ctx** out) {
  if (!cfg || !out) return DM0_EINVAL;
  *out = nullptr;
  std::string why;
  if (!cfg_ok(*cfg, &why)) return DM0_ESHAPE;
  dm0_ctx* c = new dm0_ctx();
  c->cfg = *cfg;
  const dm0_config& g = c->cfg;
  auto bail = [&](dm0_status st) {
    dm0_destroy(c);
    return st;
  };
  if (cudaGetDevice(&c->device) != cudaSuccess) return bail(DM0_ECUDA);
  cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
  if (const char* e = std::getenv("DM0_NO_PDL")) c->use_pdl = e[0] == '0';
  if (const char* e = std::getenv("DM0_NO_GRAPH")) c->use_graph = e[0] == '0';
  if (const char* e = std::getenv("DM0_NO_PERSIST")) c->use_persist = e[0] == '0';
  if (const char* e = std::getenv("DM0_PERSIST_SPLITS")) c->persist_splits = std::max(1, std::atoi(e));
  if (const char* e = std::getenv("DM0_PERSIST_FASTBAR")) c->persist_fast_bar = e[0] != '0';
  if (const char* e = std::getenv("DM0_QKV_EPI")) c->qkv_epi4 = std::atoi(e) != 8;
  if (const char* e = std::getenv("DM0_RASTER_BAND")) c->raster_band_override = std::max(0, std::atoi(e));

  // weights: one allocation, 256-byte aligned sub-buffers
  size_t total = 0;
  std::vector<size_t> offs;
  auto take = [&](size_t bytes) {
    offs.push_back(total);
    total += align256(bytes);
  };
  // the four matrices of a branch are each stacked over the layers ([L][rows][cols], no padding), so
  // one 2-D TMA descriptor per matrix type covers every layer
  const size_t Lz = static_cast<size_t>(g.layers);
  for (int br = 0; br < 2; ++br) {
    const size_t H = hidden_of(g, br), I = inter_of(g, br);
    take(Lz * 2 * qkv_rows(g) * H);
    take(Lz * 2 * H * g.n_q * g.head_dim);
    take(Lz * 2 * 2 * I * H);
    take(Lz * 2 * H * I);
    for (int l = 0; l < g.layers; ++l) {
      take(4 * H);
      take(4 * g.head_dim);
      take(4 * g.head_dim);
      take(4 * H);
    }
  }
  take(2 * g.hidden_a * g.action_dim);
  take(4 * g.hidden_a);
  take(4 * g.hidden_a);
  take(2 * g.action_dim * g.hidden_a);
  take(4 * g.action_dim);
  uint8_t* wb = nullptr;
  if (dalloc(c, &wb, total) != DM0_OK) return bail(DM0_ENOMEM);
  c->wbuf = wb;
  size_t k = 0;
  for (int br = 0; br < 2; ++br) {
    const size_t H = hidden_of(g, br), I = inter_of(g, br);
    c->lw_store[br].resize(g.layers);
    bf16* wqkv0 = reinterpret_cast<bf16*>(wb + offs[k++]);
    bf16* wo0 = reinterpret_cast<bf16*>(wb + offs[k++]);
    bf16* wgu0 = reinterpret_cast<bf16*>(wb + offs[k++]);
    bf16* wd0 = reinterpret_cast<bf16*>(wb + offs[k++]);
    for (int l = 0; l < g.layers; ++l) {
      LayerW& w = c->lw_store[br][l];
      w.wqkv = wqkv0 + l * qkv_rows(g) * H;
      w.wo = wo0 + l * H * g.n_q * g.head_dim;
      w.wgu = wgu0 + l * 2 * I * H;
      w.wd = wd0 + l * H * I;
      w.attn_norm = reinterpret_cast<float*>(wb + offs[k++]);
      w.q_norm = reinterpret_cast<float*>(wb + offs[k++]);
      w.k_norm = reinterpret_cast<float*>(wb + offs[k++]);
      w.mlp_norm = reinterpret_cast<float*>(wb + offs[k++]);
    }
    c->lw[br] = c->lw_store[br].data();
  }
  c->W_in = reinterpret_cast<bf16*>(wb + offs[k++]);
  c->b_in = reinterpret_cast<float*>(wb + offs[k++]);
  c->final_norm = reinterpret_cast<float*>(wb + offs[k++]);
  c->W_out = reinterpret_cast<bf16*>(wb + offs[k++]);
  c->b_out = reinterpret_cast<float*>(wb + offs[k++]);

  if (g.time_mod) {
    const size_t Ha = g.hidden_a, R = (6 * Lz + 2) * Ha;
    if (dalloc(c, &c->tm_W_ti, Ha * Ha) != DM0_OK || dalloc(c, &c->tm_W_to, Ha * Ha) != DM0_OK ||
        dalloc(c, &c->tm_Wmod, R * Ha) != DM0_OK || dalloc(c, &c->tm_b_ti, Ha) != DM0_OK ||
        dalloc(c, &c->tm_b_to, Ha) != DM0_OK || dalloc(c, &c->tm_bmod, R) != DM0_OK)
      return bail(DM0_ENOMEM);
  }

  const size_t D = g.head_dim, qd = g.n_q * D;
  const size_t Mp = static_cast<size_t>(g.max_batch) * g.max_prefix;
  const size_t Ms = static_cast<size_t>(g.max_batch) * g.chunk;
  const size_t plane = static_cast<size_t>(g.layers) * g.max_batch * g.n_kv * g.max_prefix * D;
  dm0_status st = DM0_OK;
  auto A = [&](dm0_status s2) {
    if (st == DM0_OK) st = s2;
  };
  A(dalloc(c, &c->kplane, plane));
  A(dalloc(c, &c->vplane, plane));
  A(dalloc(c, &c->h_v, Mp * g.hidden_v));
  A(dalloc(c, &c->xn_v, Mp * g.hidden_v));
  A(dalloc(c, &c->q_v, Mp * qd));
  A(dalloc(c, &c->o_v, Mp * qd));
  A(dalloc(c, &c->act_v, Mp * g.inter_v));
  A(dalloc(c, &c->ssq_v, Mp * 2 * (g.hidden_v / 64)));   // [attention, MLP norm][H / 64 groups][rows]
  A(dalloc(c, &c->h_a, Ms * g.hidden_a));
  A(dalloc(c, &c->xn_a, Ms * g.hidden_a));
  A(dalloc(c, &c->q_a, Ms * qd));
  A(dalloc(c, &c->o_a, Ms * qd));
  A(dalloc(c, &c->act_a, Ms * g.inter_a));
  A(dalloc(c, &c->ssq_a, Ms * 2 * (g.hidden_a / 64)));
  A(dalloc(c, &c->x, Ms * g.action_dim));
  A(dalloc(c, &c->k_s, Ms * g.n_kv * D));
  A(dalloc(c, &c->v_s, Ms * g.n_kv * D));
  size_t widest = qkv_rows(g);
  for (int br = 0; br < 2; ++br) widest = std::max(widest, static_cast<size_t>(2 * inter_of(g, br)));
  c->acc_elems = 128 * widest;
  A(dalloc(c, &c->acc, c->acc_elems));
  A(dalloc(c, &c->gcount, 1024));
  const int G = g.n_q / g.n_kv;
  c->acount_n = g.max_batch * g.n_kv * ((G * std::max(g.max_prefix, g.chunk) + 127) / 128) + 64;
  A(dalloc(c, &c->acount, c->acount_n));
  A(dalloc(c, &c->part_o, static_cast<size_t>(kPartSlots) * 128 * D));
  A(dalloc(c, &c->part_ml, static_cast<size_t>(kPartSlots) * 128));
  const int max_pos = g.max_prefix + g.chunk;
  A(dalloc(c, &c->rope, static_cast<size_t>(max_pos) * D / 2));
  A(dalloc(c, &c->rope_t, static_cast<size_t>(max_pos) * D / 2));
  c->rope_max_pos = max_pos;
  A(dalloc(c, &c->d_err, 1));
  A(dalloc(c, &c->stage_prefix, Mp * g.hidden_v));
  A(dalloc(c, &c->pacc_qkv, static_cast<size_t>(64) * qkv_rows(g)));
  A(dalloc(c, &c->pacc_gu, static_cast<size_t>(64) * 2 * g.inter_a));
  A(dalloc(c, &c->pssq, 128));
  A(dalloc(c, &c->psync, 2 + g.n_kv));
  A(dalloc(c, &c->pkv_sfx, static_cast<size_t>(g.n_kv) * 2 * 64 * 128));
  if (const char* e = std::getenv("DM0_ATTN_TRACE")) {
    if (e[0] == '1') A(dalloc(c, &c->atrace, static_cast<size_t>(kPartSlots) * dm0::kAttnTraceBlocks * 4));
  }
  if (const char* e = std::getenv("DM0_GEMM_TRACE")) {
    if (e[0] == '1')
      A(dalloc(c, &c->gtrace, static_cast<size_t>(kGemmTraceLaunches) * c->num_sms * dm0::kGemmTraceSlots));
  }
  if (const char* e = std::getenv("DM0_PERSIST_TRACE")) {
    if (e[0] == '1') {
      c->ptrace_steps = 16;
      A(dalloc(c, &c->ptrace, static_cast<size_t>(1 + c->ptrace_steps * (5 * g.layers + 1)) * c->num_sms * dm0::kPdTraceSlots));
    }
  }
  if (st != DM0_OK) return bail(st);
  if (cudaMemset(c->acc, 0, c->acc_elems * 4) != cudaSuccess || cudaMemset(c->gcount, 0, 1024 * 4) != cudaSuccess ||
      cudaMemset(c->acount, 0, c->acount_n * 4) != cudaSuccess || cudaMemset(c->d_err, 0, 4) != cudaSuccess)
    return bail(DM0_ECUDA);
  const int nrope = max_pos * static_cast<int>(D / 2);
  dm0::rope_table_kernel<<<(nrope + 255) / 256, 256>>>(c->rope, c->rope_t, max_pos, static_cast<int>(D / 2),
                                                       std::log(static_cast<double>(g.rope_theta)));
  if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return bail(DM0_ECUDA);
  if (cudaStreamCreateWithFlags(&c->cap_stream, cudaStreamNonBlocking) != cudaSuccess) return bail(DM0_ECUDA);

  auto smem_attr = [&](auto kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
  };
  bool ok = smem_attr(dm0::gemm_tc_kernel<64, kGemmStages>, dm0::GemmSmem<64, kGemmStages>::kBytes) &&
            smem_attr(dm0::gemm_tc_kernel<128, kGemmStages>, dm0::GemmSmem<128, kGemmStages>::kBytes) &&
            smem_attr(dm0::gemm_tc_kernel<256, kGemmStages>, dm0::GemmSmem<256, kGemmStages>::kBytes) &&
            smem_attr(dm0::gemm_tc_persistent<64, 8>, dm0::PGemmSmem<64, 8>::kBytes) &&
            smem_attr(dm0::gemm_tc_persistent<128, 6>, dm0::PGemmSmem<128, 6>::kBytes) &&
            smem_attr(dm0::gemm_tc_persistent<256, 4>, dm0::PGemmSmem<256, 4>::kBytes) &&
            smem_attr(dm0::gemm_tc_persistent<256, 4, false, 4>, dm0::PGemmSmem<256, 4, 4>::kBytes) &&
            smem_attr(dm0::gemm_tc_persistent<128, 6, false, 4>, dm0::PGemmSmem<128, 6, 4>::kBytes) &&
            smem_attr(dm0::gemm_tc_persistent<64, 8, true>, dm0::PGemmSmem<64, 8>::kBytes) &&
            smem_attr(dm0::gemm_tc_persistent<128, 6, true>, dm0::PGemmSmem<128, 6>::kBytes) &&
            smem_attr(dm0::gemm_tc_persistent<256, 4, true>, dm0::PGemmSmem<256, 4>::kBytes) &&
            smem_attr(dm0::attn_kernel<128>, dm0::AttnSmem<128>::kBytes) &&
            smem_attr(dm0::attn_kernel<64>, dm0::AttnSmem<64>::kBytes) &&
            smem_attr(dm0::attn_kernel<32>, dm0::AttnSmem<32>::kBytes) &&
            smem_attr(dm0::fa_tc_kernel<2, 1>, dm0::FaSmemT<2, 1>::kBytes) &&
            smem_attr(dm0::fa_tc_kernel<dm0::kFaDeepStages, 2>, dm0::FaSmemT<dm0::kFaDeepStages, 2>::kBytes) &&
            smem_attr(dm0::denoise_persistent_kernel<false>, dm0::PdSmem::kBytes) &&
            smem_attr(dm0::denoise_persistent_kernel<true>, dm0::PdSmem::kBytes) &&
            smem_attr(dm0::train_attn_fwd_kernel, 100 * 1024) && smem_attr(dm0::train_attn_bwd_kernel, 200 * 1024) &&
            smem_attr(dm0::fa_bwd_kernel, dm0::FaBwdSmem::kBytes);
  if (!ok) return bail(DM0_ECUDA);
  *out = c;
  return DM0_OK;
}

dm0_status dm0_load_weights(dm0_ctx* c, const void* blob, size_t bytes) {
  if (!c || !blob) return fail(c, DM0_EINVAL, "null context or blob");
  const dm0_config& g = c->cfg;
  if (bytes != blob_bytes(g))
    return fail(c, DM0_ESHAPE, "blob is " + std::to_string(bytes) + " bytes, expected " + std::to_string(blob_bytes(g)));
  const uint8_t* p = static_cast<const uint8_t*>(blob);
  auto put = [&](void* dst, size_t n) -> dm0_status {
    CK(cudaMemcpy(dst, p, n, cudaMemcpyHostToDevice));
    p += n;
    return DM0_OK;
  };
  const size_t D = g.head_dim;
  for (int br = 0; br < 2; ++br) {
    const size_t H = hidden_of(g, br), I = inter_of(g, br);
    const size_t qd = g.n_q * D, kvd = g.n_kv * D;
    for (int l = 0; l < g.layers; ++l) {
      const LayerW& w = c->lw[br][l];
      TRY(put(w.attn_norm, 4 * H));
      TRY(put(w.wqkv, 2 * qd * H));
      TRY(put(w.wqkv + qd * H, 2 * kvd * H));
      TRY(put(w.wqkv + (qd + kvd) * H, 2 * kvd * H));
      TRY(put(w.q_norm, 4 * D));
      TRY(put(w.k_norm, 4 * D));
      TRY(put(w.wo, 2 * H * qd));
      TRY(put(w.mlp_norm, 4 * H));
      // gate/up interleaved in 64-row blocks: rows [128j, 128j+64) gate block j, [128j+64, 128j+128) up block j
      for (int part = 0; part < 2; ++part) {
        CK(cudaMemcpy2D(w.wgu + part * 64 * H, 128 * H * 2, p, 64 * H * 2, 64 * H * 2, I / 64,
                        cudaMemcpyHostToDevice));
        p += 2 * I * H;
      }
      TRY(put(w.wd, 2 * H * I));
    }
  }
  const size_t Ha = g.hidden_a, Ad = g.action_dim;
  TRY(put(c->W_in, 2 * Ha * Ad));
  TRY(put(c->b_in, 4 * Ha));
  TRY(put(c->final_norm, 4 * Ha));
  TRY(put(c->W_out, 2 * Ad * Ha));
  TRY(put(c->b_out, 4 * Ad));
  if (g.time_mod) {   // the modulators' rows go to one stacked matrix: [l][attention 3Ha | MLP 3Ha], final 2Ha
    const size_t L = g.layers;
    TRY(put(c->tm_W_ti, 2 * Ha * Ha));
    TRY(put(c->tm_b_ti, 4 * Ha));
    TRY(put(c->tm_W_to, 2 * Ha * Ha));
    TRY(put(c->tm_b_to, 4 * Ha));
    TRY(put(c->tm_Wmod + 6 * L * Ha * Ha, 2 * 2 * Ha * Ha));
    TRY(put(c->tm_bmod + 6 * L * Ha, 4 * 2 * Ha));
    for (size_t l = 0; l < L; ++l) {
      for (size_t part = 0; part < 2; ++part) {
        TRY(put(c->tm_Wmod + (6 * l + 3 * part) * Ha * Ha, 2 * 3 * Ha * Ha));
        TRY(put(c->tm_bmod + (6 * l + 3 * part) * Ha, 4 * 3 * Ha));
      }
    }
  }
  c->weights_loaded = true;
  c->train_wt_ok = false;   // the training step's transposed weights are rebuilt on its next call
  if (c->fp8_mlp) {   // keep the FP8 copies in step with the new weights
    TRY(pack_fp8_weights(c, nullptr));
    CK(cudaStreamSynchronize(nullptr));
  }
  return DM0_OK;
}

dm0_status dm0_set_prefix_fp8(dm0_ctx* c, int enable, void* stream) {
  if (!c) return DM0_EINVAL;
  if (!enable) {
    c->fp8_mlp = false;
    return DM0_OK;
  }
  if (!c->weights_loaded) return fail(c, DM0_ESTATE, "load the weights before enabling the FP8 prefix MLP");
  const dm0_config& g = c->cfg;
  if (g.hidden_v % 128 != 0 || g.inter_v % 128 != 0)
    return fail(c, DM0_ESHAPE, "the FP8 prefix MLP needs hidden_v and inter_v multiples of 128");
  TRY(ensure_fp8(c));
  TRY(pack_fp8_weights(c, static_cast<cudaStream_t>(stream)));
  c->fp8_mlp = true;
  return DM0_OK;
}

dm0_status dm0_prefill(dm0_ctx* c, const void* prefix_emb, int B, int P, void* stream) {
  if (!c || !prefix_emb) return fail(c, DM0_EINVAL, "null context or prefix");
  if (!c->weights_loaded) return fail(c, DM0_ESTATE, "weights not loaded");
  if (B < 1 || B > c->cfg.max_batch || P < 1 || P > c->cfg.max_prefix)
    return fail(c, DM0_ESHAPE, "B or P outside the context capacity");
  c->kv_B = 0;
  TRY(enqueue_prefill(c, static_cast<cudaStream_t>(stream), prefix_emb, B, P));
  c->kv_B = B;
  c->kv_P = P;
  return DM0_OK;
}

dm0_status dm0_prepare(dm0_ctx* c, int B, int P, int steps) {
  if (!c) return DM0_EINVAL;
  if (!c->weights_loaded) return fail(c, DM0_ESTATE, "weights not loaded");
  const dm0_config& g = c->cfg;
  if (B < 1 || B > g.max_batch || P < 1 || P > g.max_prefix || steps < 1 || steps > 1000)
    return fail(c, DM0_ESHAPE, "B, P or steps outside the context capacity");
  if (g.time_mod) TRY(tmod_tables(c, steps));
  const int kb = c->kv_B, kp = c->kv_P;
  c->kv_B = B;
  c->kv_P = P;
  dm0_status st = DM0_OK;
  dm0::PdArgs pa;
  std::string why;
  if (!persist_plan(c, steps, nullptr, &pa, &why) && c->use_graph) {   // the persistent loop needs no capture
    const dm0_ctx::Graph* gr = nullptr;
    st = denoise_graph(c, steps, &gr);
  }
  c->kv_B = kb;
  c->kv_P = kp;
  return st;
}

dm0_status dm0_kv_view(dm0_ctx* c, void** k, void** v) {
  if (!c || !k || !v) return fail(c, DM0_EINVAL, "null argument");
  *k = c->kplane;
  *v = c->vplane;
  return DM0_OK;
}

dm0_status dm0_kv_commit(dm0_ctx* c, int B, int P) {
  if (!c) return DM0_EINVAL;
  if (B < 1 || B > c->cfg.max_batch || P < 1 || P > c->cfg.max_prefix)
    return fail(c, DM0_ESHAPE, "B or P outside the context capacity");
  c->kv_B = B;
  c->kv_P = P;
  return DM0_OK;
}

dm0_status dm0_denoise(dm0_ctx* c, const float* noise, int steps, float* actions, float* vel, void* stream) {
  if (!c || !noise || !actions) return fail(c, DM0_EINVAL, "null argument");
  if (!c->weights_loaded) return fail(c, DM0_ESTATE, "weights not loaded");
  if (c->kv_B == 0) return fail(c, DM0_ESTATE, "no KV cache: call dm0_prefill or dm0_kv_commit first");
  if (steps < 1 || steps > 1000) return fail(c, DM0_ESHAPE, "steps must be in [1, 1000]");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(c->kv_B) * c->cfg.chunk * c->cfg.action_dim * sizeof(float);
  CK(cudaMemcpyAsync(c->x, noise, bytes, cudaMemcpyDeviceToDevice, s));
  TRY(denoise_from_x(c, s, steps, vel));
  CK(cudaMemcpyAsync(actions, c->x, bytes, cudaMemcpyDeviceToDevice, s));
  return DM0_OK;
}

dm0_status dm0_infer_host(dm0_ctx* c, const void* prefix_emb, const float* noise, int B, int P, int steps,
                          float* actions, void* stream) {
  if (!c || !prefix_emb || !noise || !actions) return fail(c, DM0_EINVAL, "null argument");
  if (!c->weights_loaded) return fail(c, DM0_ESTATE, "weights not loaded");
  if (B < 1 || B > c->cfg.max_batch || P < 1 || P > c->cfg.max_prefix || steps < 1 || steps > 1000)
    return fail(c, DM0_ESHAPE, "B, P or steps outside the context capacity");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t pbytes = static_cast<size_t>(B) * P * c->cfg.hidden_v * 2;
  const size_t xbytes = static_cast<size_t>(B) * c->cfg.chunk * c->cfg.action_dim * sizeof(float);
  CK(cudaMemcpyAsync(c->stage_prefix, prefix_emb, pbytes, cudaMemcpyHostToDevice, s));
  CK(cudaMemcpyAsync(c->x, noise, xbytes, cudaMemcpyHostToDevice, s));
  c->kv_B = 0;
  TRY(enqueue_prefill(c, s, c->stage_prefix, B, P));
  c->kv_B = B;
  c->kv_P = P;
  TRY(denoise_from_x(c, s, steps, nullptr));
  CK(cudaMemcpyAsync(actions, c->x, xbytes, cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  return DM0_OK;
}

dm0_status dm0_merged_layer(dm0_ctx* c, int layer, const float* h_prefix, const float* h_suffix, int B, int P,
                            float* out_prefix, float* out_suffix, void* k_out, void* v_out, void* stream) {
  if (!c || !h_prefix || !h_suffix || !out_prefix || !out_suffix || !k_out || !v_out)
    return fail(c, DM0_EINVAL, "null argument");
  if (!c->weights_loaded) return fail(c, DM0_ESTATE, "weights not loaded");
  const dm0_config& g = c->cfg;
  if (g.time_mod) return fail(c, DM0_EINVAL, "the merged layer has no flow time: it covers the DM0 layer only");
  if (layer < 0 || layer >= g.layers || B < 1 || B > g.max_batch || P < 1 || P > g.max_prefix)
    return fail(c, DM0_ESHAPE, "layer, B or P outside the context capacity");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int Mp = B * P, S = g.chunk, Ms = B * S;
  bf16* kp = static_cast<bf16*>(k_out);
  bf16* vp = static_cast<bf16*>(v_out);
  c->pdl_ok = false;
  const int nsv = g.hidden_v / 64, nsa = g.hidden_a / 64;   // sum-of-squares groups per row
  TRY(rows_prep(c, s, h_prefix, 0, c->h_v, c->xn_v, c->lw[0][layer].attn_norm, c->ssq_v, nsv, Mp, g.hidden_v));
  TRY(rows_prep(c, s, h_suffix, 0, c->h_a, c->xn_a, c->lw[1][layer].attn_norm, c->ssq_a, nsa, Ms, g.hidden_a));
  TRY(layer_qkv(c, s, 0, layer, c->xn_v, c->ssq_v, Mp, P, 0, c->q_v, kp, vp));
  TRY(layer_qkv(c, s, 1, layer, c->xn_a, c->ssq_a, Ms, S, P, c->q_a, c->k_s, c->v_s));
  // the block mask: prefix rows see the prefix; suffix rows see prefix and suffix
  TRY(run_attn(c, s, c->q_v, P, kp, vp, P, nullptr, nullptr, 0, c->o_v, B, 1, 0));
  TRY(run_attn(c, s, c->q_a, S, kp, vp, P, c->k_s, c->v_s, S, c->o_a, B, 0, 0));
  TRY(layer_rest(c, s, 0, layer, Mp, c->h_v, c->xn_v, c->o_v, c->act_v, c->ssq_v + static_cast<size_t>(nsv) * Mp,
                 nullptr, nullptr));
  TRY(layer_rest(c, s, 1, layer, Ms, c->h_a, c->xn_a, c->o_a, c->act_a, c->ssq_a + static_cast<size_t>(nsa) * Ms,
                 nullptr, nullptr));
  CK(cudaMemcpyAsync(out_prefix, c->h_v, static_cast<size_t>(Mp) * g.hidden_v * 4, cudaMemcpyDeviceToDevice, s));
  CK(cudaMemcpyAsync(out_suffix, c->h_a, static_cast<size_t>(Ms) * g.hidden_a * 4, cudaMemcpyDeviceToDevice, s));
  return DM0_OK;
}

dm0_status dm0_op_gemm(dm0_ctx* c, const void* A, const void* B, float* C, int M, int N, int K, int swap,
                       int splits, void* stream) {
  if (!c || !A || !B || !C) return fail(c, DM0_EINVAL, "null argument");
  if (M < 1 || N < 1 || K < 64 || K % 64 != 0 || splits < 1) return fail(c, DM0_ESHAPE, "bad GEMM shape");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  c->pdl_ok = false;
  GemmArgs g = base_args(c);
  g.mode = dm0::kModeStoreF32;
  if (swap) {
    if (M % 128 != 0 || N > 128) return fail(c, DM0_ESHAPE, "swap GEMM needs M % 128 == 0 and N <= 128");
    g.acc = C;
    g.ld_acc = M;
    return run_gemm(c, s, static_cast<const bf16*>(B), N, K, static_cast<const bf16*>(A), M, g, 1, splits);
  }
  if (N % 128 != 0 || splits != 1) return fail(c, DM0_ESHAPE, "GEMM needs N % 128 == 0 and splits == 1");
  g.out_f32 = C;
  return run_gemm(c, s, static_cast<const bf16*>(A), M, K, static_cast<const bf16*>(B), N, g, 0, 1);
}

size_t dm0_grad_floats(const dm0_config* cfg) { return cfg ? grad_floats(*cfg) : 0; }

dm0_status dm0_train_step(dm0_ctx* c, const float* a, const float* eps, const float* t, const uint8_t* mask,
                          float* loss, float* grads, float* kv_grads, void* stream) {
  if (!c || !a || !eps || !t || !mask || !loss || !grads) return fail(c, DM0_EINVAL, "null argument");
  if (!c->weights_loaded) return fail(c, DM0_ESTATE, "weights not loaded");
  if (c->kv_B < 1) return fail(c, DM0_ESTATE, "no prefix cache: call dm0_prefill or dm0_kv_commit first");
  const dm0_config& g = c->cfg;
  if (g.time_mod) return fail(c, DM0_EINVAL, "the training step covers the DM0 action expert (time_mod = 0)");
  if (g.chunk * g.head_dim > 32 * 256) return fail(c, DM0_ESHAPE, "chunk * head_dim must be <= 8192");
  if (reinterpret_cast<uintptr_t>(grads) % 16 != 0) return fail(c, DM0_EINVAL, "grads must be 16-byte aligned");
  TRY(train_buffers(c));
  return enqueue_train(c, static_cast<cudaStream_t>(stream), a, eps, t, mask, loss, grads, kv_grads);
}

dm0_status dm0_op_quant_e4m3(dm0_ctx* c, const void* x, int x_f32, int rows, int cols, const float* gain,
                             const float* ssq, void* codes, float* scales, void* stream) {
  if (!c || !x || !codes || !scales) return fail(c, DM0_EINVAL, "null argument");
  if (rows < 1 || cols < 8 || cols % 8 != 0) return fail(c, DM0_ESHAPE, "quantisation needs rows >= 1, cols % 8 == 0");
  if (reinterpret_cast<uintptr_t>(x) % 16 != 0 || reinterpret_cast<uintptr_t>(codes) % 8 != 0 ||
      (gain && reinterpret_cast<uintptr_t>(gain) % 16 != 0))
    return fail(c, DM0_EINVAL, "x and gain must be 16-byte and codes 8-byte aligned");
  c->pdl_ok = false;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* q = static_cast<uint8_t*>(codes);
  if (x_f32) return quant_rows(c, s, static_cast<const float*>(x), rows, cols, q, scales, gain, ssq);
  return quant_rows(c, s, static_cast<const bf16*>(x), rows, cols, q, scales, gain, ssq);
}

dm0_status dm0_op_gemm_e4m3(dm0_ctx* c, const void* A, const float* sa, const void* B, const float* sb, float* C,
                            int M, int N, int K, void* stream) {
  if (!c || !A || !sa || !B || !sb || !C) return fail(c, DM0_EINVAL, "null argument");
  if (M < 1 || N < 128 || N % 128 != 0 || K < 128 || K % 128 != 0)
    return fail(c, DM0_ESHAPE, "FP8 GEMM needs M >= 1, N % 128 == 0, K % 128 == 0");
  if (reinterpret_cast<uintptr_t>(sb) % 16 != 0) return fail(c, DM0_EINVAL, "sb must be 16-byte aligned");
  c->pdl_ok = false;
  GemmArgs g = base_args(c);
  g.mode = dm0::kModeStoreF32;
  g.out_f32 = C;
  return run_gemm_e4m3(c, static_cast<cudaStream_t>(stream), static_cast<const uint8_t*>(A), sa, M, K,
                       static_cast<const uint8_t*>(B), sb, N, g);
}

dm0_status dm0_op_attention(dm0_ctx* c, const void* q, const void* ka, const void* va, int Ta, const void* kb,
                            const void* vb, int Tb, void* o, int B, int Tq, int splits, void* stream) {
  if (!c || !q || !ka || !va || !o || (Tb > 0 && (!kb || !vb))) return fail(c, DM0_EINVAL, "null argument");
  if (B < 1 || Tq < 1 || Ta < 1 || Tb < 0 || splits < 1) return fail(c, DM0_ESHAPE, "bad attention shape");
  const int G = c->cfg.n_q / c->cfg.n_kv;
  if (splits > 1 && B * c->cfg.n_kv * ((G * Tq + 127) / 128) > c->acount_n)
    return fail(c, DM0_ESHAPE, "too many row tiles for a split launch");
  c->pdl_ok = false;
  return run_attn(c, static_cast<cudaStream_t>(stream), static_cast<const bf16*>(q), Tq, static_cast<const bf16*>(ka),
                  static_cast<const bf16*>(va), Ta, static_cast<const bf16*>(kb), static_cast<const bf16*>(vb), Tb,
                  static_cast<bf16*>(o), B, splits, 0);
}

dm0_status dm0_debug_view(dm0_ctx* c, const char* name, void** ptr) {
  if (!c || !name || !ptr) return fail(c, DM0_EINVAL, "null argument");
  const std::map<std::string, void*> bufs = {
      {"h_v", c->h_v},     {"xn_v", c->xn_v},   {"q_v", c->q_v},     {"o_v", c->o_v},     {"act_v", c->act_v},
      {"ssq_v", c->ssq_v}, {"h_a", c->h_a},     {"xn_a", c->xn_a},   {"q_a", c->q_a},     {"o_a", c->o_a},
      {"act_a", c->act_a}, {"ssq_a", c->ssq_a}, {"x", c->x},         {"k_s", c->k_s},     {"v_s", c->v_s},
      {"loop_trace", c->ptrace}, {"gemm_trace", c->gtrace}, {"attn_trace", c->atrace}, {"tm_mod", c->tm_mod}, {"tm_bqkv", c->tm_bqkv}, {"tm_bgu", c->tm_bgu}};
  auto it = bufs.find(name);
  if (it == bufs.end()) return fail(c, DM0_EINVAL, std::string("unknown buffer ") + name);
  *ptr = it->second;
  return DM0_OK;
}

uint64_t dm0_launch_count(const dm0_ctx* c) { return c ? c->launches : 0; }

dm0_status dm0_probe(dm0_ctx* c, int site_mask) {
  if (!c) return DM0_EINVAL;
  if (site_mask < 0 || site_mask >= (1 << DM0_SITE_COUNT)) return fail(c, DM0_EINVAL, "unknown probe site");
  c->probe_mask = site_mask;
  c->probe_used = 0;
  c->probe_recs.clear();
  return DM0_OK;
}

dm0_status dm0_probe_read(dm0_ctx* c, int site, int* launches, double* total_ms) {
  if (!c || !launches || !total_ms) return fail(c, DM0_EINVAL, "null argument");
  double tot = 0.0;
  int n = 0;
  for (const auto& r : c->probe_recs) {
    if (r.site != site) continue;
    CK(cudaEventSynchronize(c->probe_ev[r.e1]));
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, c->probe_ev[r.e0], c->probe_ev[r.e1]));
    tot += ms;
    ++n;
  }
  *launches = n;
  *total_ms = tot;
  return DM0_OK;
}

dm0_status dm0_attention_noalloc(const void* q, const void* ka, const void* va, int Ta, const void* kb, const void* vb,
                                 int Tb, void* o, int B, int Tq, int n_q, int n_kv, int head_dim, int splits,
                                 void* stream) {
  if (!q || !ka || !va || !o || (Tb > 0 && (!kb || !vb))) return DM0_EINVAL;
  if (B < 1 || Tq < 1 || Ta < 1 || Tb < 0 || splits < 1 || n_q < 1 || n_kv < 1 || n_q % n_kv != 0)
    return DM0_ESHAPE;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return DM0_ESHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DM0_ECUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return DM0_ECUDA;
  float* base = nullptr;
  TRY(noalloc_setup(dev, &base));
  const int G = n_q / n_kv;
  const long long tiles = (static_cast<long long>(G) * Tq + 127) / 128;
  const long long groups = static_cast<long long>(B) * n_kv;
  const int nblk = (Ta + Tb + 63) / 64;
  if (tiles > 65535 || groups > 65535) return DM0_ESHAPE;
  if (splits > nblk) splits = nblk;
  const int bps = (nblk + splits - 1) / splits;
  splits = (nblk + bps - 1) / bps;
  if (splits > 1 && groups * tiles * splits > kNoAllocSlots) return DM0_ESHAPE;   // beyond the static scratch
  const int smem_bytes = head_dim == 128 ? dm0::AttnSmem<128>::kBytes
                                         : (head_dim == 64 ? dm0::AttnSmem<64>::kBytes : dm0::AttnSmem<32>::kBytes);
  if (splits > 1 && splits * 128 * 8 > smem_bytes) return DM0_ESHAPE;   // the combine's (m, l) in shared memory
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* counters = reinterpret_cast<int*>(base + kNoAllocOFloats + kNoAllocMlFloats);
  if (splits > 1 && cudaMemsetAsync(counters, 0, kNoAllocCounters * sizeof(int), s) != cudaSuccess)
    return DM0_ECUDA;
  AttnArgs a{};
  a.q = static_cast<const bf16*>(q);
  a.seq_q = Tq;
  a.ka = static_cast<const bf16*>(ka);
  a.va = static_cast<const bf16*>(va);
  a.len_a = Ta;
  a.kb = static_cast<const bf16*>(kb);
  a.vb = static_cast<const bf16*>(vb);
  a.len_b = Tb;
  a.o = static_cast<bf16*>(o);
  a.n_q = n_q;
  a.n_kv = n_kv;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(head_dim)));
  a.blocks_per_split = bps;
  a.a_stable = 0;
  a.part_o = base;
  a.part_ml = reinterpret_cast<float2*>(base + kNoAllocOFloats);
  a.counters = counters;
  a.err = nullptr;
  const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(groups), splits);
  switch (head_dim) {
    case 128:
      dm0::attn_kernel<128><<<grid, dm0::kAttnThreads, dm0::AttnSmem<128>::kBytes, s>>>(a);
      break;
    case 64:
      dm0::attn_kernel<64><<<grid, dm0::kAttnThreads, dm0::AttnSmem<64>::kBytes, s>>>(a);
      break;
    default:
      dm0::attn_kernel<32><<<grid, dm0::kAttnThreads, dm0::AttnSmem<32>::kBytes, s>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? DM0_OK : DM0_ECUDA;
}

dm0_status dm0_selftest_timeout(dm0_ctx* c, int limit_us, void* stream) {
  if (!c) return DM0_EINVAL;
  if (limit_us < 1 || limit_us > 1000000) return fail(c, DM0_ESHAPE, "limit_us must be in [1, 1e6]");
  c->pdl_ok = false;
  dm0::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      c->d_err, static_cast<unsigned long long>(limit_us) * 1000ull);
  CK(cudaGetLastError());
  return DM0_OK;
}

dm0_status dm0_sync(dm0_ctx* c, void* stream) {
  if (!c) return DM0_EINVAL;
  CK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int e = 0;
  CK(cudaMemcpy(&e, c->d_err, 4, cudaMemcpyDeviceToHost));
  if (e) return fail(c, DM0_EDEVICE, "device error word " + std::to_string(e));
  return DM0_OK;
}

int dm0_device_error(const dm0_ctx* c) {
  if (!c) return -1;
  int e = 0;
  if (cudaMemcpy(&e, c->d_err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
  return e;
}

dm0_status dm0_clear_error(dm0_ctx* c) {
  if (!c) return DM0_EINVAL;
  CK(cudaDeviceSynchronize());
  CK(cudaMemset(c->d_err, 0, 4));
  CK(cudaMemset(c->acc, 0, c->acc_elems * 4));
  CK(cudaMemset(c->gcount, 0, 1024 * 4));
  CK(cudaMemset(c->acount, 0, c->acount_n * 4));
  CK(cudaDeviceSynchronize());
  return DM0_OK;
}

const char* dm0_last_error(const dm0_ctx* c) {
  if (!c) return "null context";
  return c->err.c_str();
}

void dm0_destroy(dm0_ctx* c) {
  if (!c) return;
  for (auto& kv : c->graphs) cudaGraphExecDestroy(kv.second.exec);
  for (cudaEvent_t e : c->probe_ev) cudaEventDestroy(e);
  if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
  for (void* p : c->allocs) cudaFree(p);
  delete c;
}

dm0_status dm0_pack_e4m3_rows(const float* x, int64_t rows, int64_t cols, uint8_t* codes, float* scales) {
  if (!x || !codes || !scales) return DM0_EINVAL;
  if (rows < 1 || cols < 1) return DM0_ESHAPE;
  for (int64_t r = 0; r < rows; ++r) {
    const float* row = x + r * cols;
    double amax = 0.0;
    for (int64_t k = 0; k < cols; ++k) {
      if (!std::isfinite(row[k])) return DM0_EINVAL;
      amax = std::max(amax, std::fabs(static_cast<double>(row[k])));
    }
    const double s = amax > 0.0 ? amax / 448.0 : 1.0;
    scales[r] = static_cast<float>(s);
    for (int64_t k = 0; k < cols; ++k) {
      const double v = static_cast<double>(row[k]) / s;
      const double a = std::fabs(v);
      // spacing 2^(e-3) with e = floor(log2 a) in [-6, 8] (below 2^-6: the subnormal spacing 2^-9)
      int e = a > 0.0 ? static_cast<int>(std::floor(std::log2(a))) : -6;
      e = std::min(8, std::max(-6, e));
      double q = std::nearbyint(std::ldexp(a, 3 - e));   // the default rounding mode: ties to even
      q = std::ldexp(q, e - 3);
      if (q > 448.0) q = 448.0;
      uint8_t bits = 0;
      if (q > 0.0) {
        if (q < 0.015625) {   // subnormal: m 2^-9, m in 1..7
          bits = static_cast<uint8_t>(std::lrint(std::ldexp(q, 9)));
        } else {              // normal: (1 + m/8) 2^E, biased exponent E + 7 in 1..15
          const int E = static_cast<int>(std::floor(std::log2(q)));
          const int m = static_cast<int>(std::lrint(std::ldexp(q, 3 - E))) - 8;
          bits = static_cast<uint8_t>(((E + 7) << 3) | m);
        }
      }
      if (std::signbit(v) && q > 0.0) bits |= 0x80;
      codes[r * cols + k] = bits;
    }
  }
  return DM0_OK;
}

}  // extern "C"
