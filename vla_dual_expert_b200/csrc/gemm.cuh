// Warp-specialised tcgen05 GEMM for the projection and SwiGLU contractions of
// the DM0 layers, with the per-layer element-wise work fused into its
// epilogue.
//
//   D[128 x BN tile] = A[M][K] * B[N][K]^T, bf16 operands staged by TMA with
//   128-byte swizzle, fp32 accumulator in TMEM.
//
// Two operand orientations:
//   normal (swap = 0): A = activations [tokens][K], B = weights [out][K];
//                      TMEM lanes = tokens.  Used when tokens > 128.
//   swap   (swap = 1): A = weights, B = activations (<= 128 tokens, padded by
//                      TMA zero fill); TMEM lanes = output features.  K is
//                      split across CTAs; partial sums are added with fp32
//                      atomics and the last CTA of each feature tile applies
//                      the epilogue.  Used for the 50-token action suffix.
//
// Warp roles (192 threads): warp 0 issues TMA, warp 1 owns TMEM and issues
// tcgen05.mma, warps 2..5 run the epilogue.  Weight tiles are requested before
// griddepcontrol.wait, so under programmatic dependent launch the weight
// stream of this GEMM overlaps the tail of the previous kernel.
#pragma once
#include "ptx.cuh"

namespace dm0 {

enum GemmMode : int {
  kModeStoreF32 = 0,  // C = acc (normal) / C += acc (swap)   -- unit tests
  kModeQKV = 1,       // scale by inv_rms, QK-RMSNorm + RoPE on q/k heads, write q / K / V (bf16)
  kModeResid = 2,     // h += acc; xn = bf16(gain_next * h); ssq_out = sum(h^2) per 64-column group
  kModeSwiGLU = 3,    // scale by inv_rms; act = silu(gate) * up (bf16); gate/up interleaved by 64 rows
};

struct GemmArgs {
  int M, N, K;
  int kb_per_split;   // 64-wide k-blocks per split
  int swap;
  int mode;
  int tokens;         // valid activation rows
  int w_stable;       // weight operand was written before the previous kernel: fetch it before the PDL wait
  int* err;           // device error word
  // input row scale: inv_rms(token) = rsqrt(sum_s ssq_in[s * ssq_stride + token] * inv_hidden + eps)
  // over the ssq_slots partial sums of squares (one per 64-column group of the residual, added in
  // slot order so the result does not depend on which CTA finished first); null -> 1
  const float* ssq_in;
  float inv_hidden, eps;
  int ssq_slots, ssq_stride;   // also the layout of ssq_out
  // split-K accumulation target (swap, QKV / SwiGLU / StoreF32): acc[token * ld_acc + feature]
  float* acc;
  int ld_acc;
  int* counters;      // one per 128-feature tile, zero between launches
  int band_m;         // persistent GEMM: m-tiles per raster band (1: n fastest; <= 0: the default)
  // persistent GEMM timeline (null: off): [CTA][kGemmTraceSlots] %globaltimer marks, see kGemmTrace*
  unsigned long long* trace;
  // kModeResid
  float* h;           // [tokens][H] fp32 residual stream
  int H;
  __nv_bfloat16* xn;  // [tokens][H] bf16(gain_next * h) for the next norm (null: skip)
  const float* gain_next;
  float* ssq_out;     // [H / 64][ssq_stride]: per 64-column group, the sum of squares of h over the
                      // group's columns (plain stores, no atomics; null: skip)
  // kModeQKV
  __nv_bfloat16* q_out;   // [tokens][n_q * head_dim]
  __nv_bfloat16* k_out;   // [B][n_kv][kv_seq][head_dim]
  __nv_bfloat16* v_out;
  const float* q_gain;
  const float* k_gain;
  int n_q, n_kv, head_dim;
  int seq_len;        // tokens per sample in this pass
  int pos_offset;     // RoPE position of each sample's first token
  int kv_seq;         // per-(sample, kv head) length of the K/V destination
  const float2* rope; // [position][head_dim/2] (cos, sin)
  const float2* rope_t;   // the same values [head_dim/2][rope_ld]: a warp's consecutive tokens read
  int rope_ld;            // one frequency as contiguous memory
  // kModeSwiGLU
  __nv_bfloat16* act; // [tokens][inter]
  int inter;
  float* act_f32;     // [tokens][inter] fp32 instead of act when not null (the FP8 MLP's down operand)
  // kModeStoreF32
  float* out_f32;     // normal: [M][N]
  // FP8 E4M3 operands (persistent normal-orientation GEMM only): the accumulator of (token, feature)
  // is multiplied by row_scale[token] * col_scale[feature] before the mode's epilogue
  const float* row_scale;   // [M] per-token activation scale
  const float* col_scale;   // [N] per-output-channel weight scale
  // time-modulated action expert (adaptive RMSNorm): null in the plain model
  const float* col_bias;    // QKV / SwiGLU: feature bias added after the pending 1/rms (the norm's shift
                            // projected through the weights)
  const float* col_gate;    // residual: per-feature gate applied to the sublayer output before the add
};

constexpr int kGemmThreads = 192;
// persistent GEMM: producer warp, MMA warp and EPI epilogue warps (4: one per TMEM lane quarter, up to
// 255 registers a thread, for the register-hungry QKV epilogue; 8: two per quarter, 168 registers)
template <int EPI>
struct PGemmWarps {
  static constexpr int kThreads = 64 + 32 * EPI;
};

// Timeline marks of the persistent GEMM, one row of kGemmTraceSlots u64 per CTA; CTA 0 also stores
// the launch shape in the last two slots ((M << 32) | N and (K << 32) | BN).
enum GemmTraceMark : int {
  kGtEntry = 0,        // thread 0 at kernel entry
  kGtSetup = 1,        // after barrier init, TMEM allocation and the setup barrier
  kGtDepWait = 2,      // producer past the dependency wait (griddepcontrol.wait)
  kGtFirstStage = 3,   // MMA warp: first k-block of the first tile landed
  kGtFirstIssued = 4,  // MMA warp: last MMA of the first tile issued
  kGtFirstAcc = 5,     // epilogue warp 2: accumulator of the first tile complete
  kGtFirstDone = 6,    // epilogue warp 2: epilogue of the first tile done
  kGtLastDone = 7,     // epilogue warp 2: epilogue of the CTA's last tile done
  kGtLastLoad = 8,     // producer: last TMA copy issued
  kGtExit = 9,         // thread 0 after the final barrier
};
constexpr int kGemmTraceSlots = 16;
__device__ __forceinline__ void gemm_mark(const unsigned long long* tr, int mark) {
  if (tr) const_cast<unsigned long long*>(tr)[blockIdx.x * kGemmTraceSlots + mark] = globaltimer();
}

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr uint32_t kA = 128 * 128;   // 128 rows x 64 bf16
  static constexpr uint32_t kB = BN * 128;
  static constexpr uint32_t kStage = kA + kB;
  static constexpr uint32_t kPipe = STAGES * kStage;
  static constexpr uint32_t kBytes = kPipe + 256 + 1024;   // + barriers + alignment slack
  static constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
};

// ---------------------------------------------------------------- epilogue of one accumulator row
//
// One thread owns one output row (a token) and walks one 128-column group of
// output features [col0, col0 + 128) in four 32-column chunks.  `load(c, v)`
// delivers the raw accumulator of chunk c: straight from TMEM (normal
// orientation: TMEM lane = token) or from the split-K scratch in L2 (swapped
// orientation, last CTA of a feature tile).  Every reduction the fused
// operations need (the head's RMSNorm, the sum of squares of the residual) is
// local to the thread, RoPE partners (d, d + D/2) sit in the same thread, and
// all loads and stores of a tile are in flight together.
//
// The TMEM loader is warp-collective: it is called for every row, valid or
// not; stores are predicated on `valid`.

__device__ __forceinline__ void st_f32x32(float* dst, const float (&v)[32]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
__device__ __forceinline__ void ld_f32x32(const float* src, float (&v)[32]) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 t = __ldcg(s4 + i);
    v[4 * i] = t.x;
    v[4 * i + 1] = t.y;
    v[4 * i + 2] = t.z;
    v[4 * i + 3] = t.w;
  }
}
__device__ __forceinline__ uint32_t bf2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}
// 32 consecutive bf16 (64 bytes, 16-byte aligned)
__device__ __forceinline__ void st_bf16x32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    d4[i] = make_uint4(bf2(v[8 * i], v[8 * i + 1]), bf2(v[8 * i + 2], v[8 * i + 3]), bf2(v[8 * i + 4], v[8 * i + 5]),
                       bf2(v[8 * i + 6], v[8 * i + 7]));
}

// Residual epilogue of the persistent (normal-orientation) GEMM with coalesced global traffic.  A
// warp's 32 tokens are TMEM lanes 32w..32w+31; for each 32-column chunk the warp passes h through a
// per-warp shared scratch, so h is read and written as whole 128-byte row pieces (4 rows per warp
// instruction) and the bf16 norm operand as 64-byte pieces (8 rows), where a thread-per-row access
// touches 32 rows per instruction.  The next chunk of h is requested before the current one is
// used.  Same results as row_epilogue's residual mode.
struct ResidScratch {
  // 32 rows x 32 fp32, 128 bytes a row, the 16-byte pieces of row r swizzled by r mod 8 so that both a
  // row-per-lane pass and a 4-rows-per-instruction pass hit every bank once per 128 bytes; the bf16
  // norm operand reuses it once h has left
  static constexpr uint32_t kBytes = 4096;
};
__device__ __forceinline__ uint32_t resid_swz(int row, int piece) {   // byte offset of 16-byte piece `piece`
  return static_cast<uint32_t>(row * 128 + ((piece ^ (row & 7)) << 4));
}

template <class Load>
__device__ __forceinline__ void resid_epilogue_warp(const GemmArgs& a, int row0, int col0, int nchunks,
                                                    uint8_t* scr, Load&& load) {
  const int lane = threadIdx.x & 31;
  const int tok = row0 + lane;
  const bool valid = tok < a.M;
  const int qr = lane >> 3, qc = lane & 7;   // h piece of this lane: row 4 i + qr, float4 qc
  float4 hn[8];
  auto fetch = [&](int c) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = row0 + 4 * i + qr;
      hn[i] = r < a.M ? __ldcg(reinterpret_cast<const float4*>(a.h + static_cast<size_t>(r) * a.H + col0 + 32 * c) + qc)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  fetch(0);
  float grp = 0.f;   // sum of squares over the current 64-column group
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    const int cc = col0 + 32 * c;
    float v[32];
    load(c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) *reinterpret_cast<float4*>(scr + resid_swz(4 * i + qr, qc)) = hn[i];
    if (c + 1 < nchunks) fetch(c + 1);
    __syncwarp();
#pragma unroll
    for (int j4 = 0; j4 < 8; ++j4) {
      float4* slot = reinterpret_cast<float4*>(scr + resid_swz(lane, j4));
      const float4 hv = *slot;
      if (a.col_gate) {
        const float4 gt = __ldg(reinterpret_cast<const float4*>(a.col_gate + cc) + j4);
        v[4 * j4] *= gt.x;
        v[4 * j4 + 1] *= gt.y;
        v[4 * j4 + 2] *= gt.z;
        v[4 * j4 + 3] *= gt.w;
      }
      v[4 * j4] += hv.x;
      v[4 * j4 + 1] += hv.y;
      v[4 * j4 + 2] += hv.z;
      v[4 * j4 + 3] += hv.w;
      *slot = make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 4 * i + qr;
      if (row0 + r < a.M)
        reinterpret_cast<float4*>(a.h + static_cast<size_t>(row0 + r) * a.H + cc)[qc] =
            *reinterpret_cast<const float4*>(scr + resid_swz(r, qc));
    }
    if (a.xn) {
      __syncwarp();   // h has been read out of the scratch
#pragma unroll
      for (int j8 = 0; j8 < 4; ++j8) {
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gain_next + cc) + 2 * j8);
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gain_next + cc) + 2 * j8 + 1);
        const float* w = v + 8 * j8;
#pragma unroll
        for (int j = 0; j < 8; ++j) grp += w[j] * w[j];
        *reinterpret_cast<uint4*>(scr + resid_swz(lane, j8)) =
            make_uint4(bf2(g0.x * w[0], g0.y * w[1]), bf2(g0.z * w[2], g0.w * w[3]), bf2(g1.x * w[4], g1.y * w[5]),
                       bf2(g1.z * w[6], g1.w * w[7]));
      }
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 8 * i + (lane >> 2), q = lane & 3;
        if (row0 + r < a.M)
          reinterpret_cast<uint4*>(a.xn + static_cast<size_t>(row0 + r) * a.H + cc)[q] =
              *reinterpret_cast<const uint4*>(scr + resid_swz(r, q));
      }
    }
    if ((c & 1) && a.ssq_out) {   // the group's partial goes to its own slot
      if (valid) a.ssq_out[static_cast<size_t>(cc >> 6) * a.ssq_stride + tok] = grp;
      grp = 0.f;
    }
    __syncwarp();   // the scratch is rewritten by the next chunk
  }
}

// `nchunks` (4, or 2 for a 64-column tile) applies to the column-independent modes (residual, store);
// QKV and SwiGLU always take a full 128-column group.
// sgain (optional): the QK-norm gains [q | k], head_dim each, staged in shared memory by the caller;
// null: read from global memory
template <bool kFromScratch, class Load>
__device__ __forceinline__ void row_epilogue(const GemmArgs& a, int tok, bool valid, int col0,
                                             Load&& load, int nchunks = 4, const float* sgain = nullptr) {
  const int D = a.head_dim;
  if (a.mode == kModeStoreF32) {
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
      float v[32];
      load(c, v);
      if (valid) st_f32x32(a.out_f32 + static_cast<size_t>(tok) * a.N + col0 + 32 * c, v);
    }
    return;
  }
  if (a.mode == kModeResid) {
    float grp = 0.f;   // sum of squares over the current 64-column group
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
      float v[32];
      load(c, v);
      if (!valid) continue;
      float* hp = a.h + static_cast<size_t>(tok) * a.H + col0 + 32 * c;
      if (!kFromScratch) {   // normal orientation: add into the residual stream here
        float hv[32];
        ld_f32x32(hp, hv);
        if (a.col_gate) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= a.col_gate[col0 + 32 * c + j];
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += hv[j];
        st_f32x32(hp, v);
      }
      if (a.xn) {
        float g[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          g[j] = a.gain_next[col0 + 32 * c + j] * v[j];
          grp += v[j] * v[j];
        }
        st_bf16x32(a.xn + static_cast<size_t>(tok) * a.H + col0 + 32 * c, g);
      }
      if ((c & 1) && a.ssq_out) {   // the group's partial goes to its own slot
        a.ssq_out[static_cast<size_t>((col0 + 32 * c) >> 6) * a.ssq_stride + tok] = grp;
        grp = 0.f;
      }
    }
    return;
  }
  // QKV and SwiGLU consume the pending RMSNorm's 1/rms of this token; with a feature bias (the
  // modulated norm's shift projected through the weights) the loader returns acc / rms + bias and the
  // code below sees a unit scale
  float s_rms = 1.f;
  if (a.ssq_in && valid) {
    float ss = 0.f;
    for (int q = 0; q < a.ssq_slots; ++q) ss += __ldcg(a.ssq_in + static_cast<size_t>(q) * a.ssq_stride + tok);
    s_rms = rsqrtf(ss * a.inv_hidden + a.eps);
  }
  const float* bias = a.col_bias;
  const float s = bias ? 1.f : s_rms;
  auto ld = [&](int c, float (&v)[32]) {
    load(c, v);
    if (bias) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = v[j] * s_rms + bias[col0 + 32 * c + j];
    }
  };
  if (a.mode == kModeSwiGLU) {
    // group = [64 gate rows | 64 up rows] of outputs [col0/2, col0/2 + 64)
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      float g[32], u[32];
      ld(c, g);
      ld(c + 2, u);
#pragma unroll
      for (int j = 0; j < 32; ++j) g[j] = silu_f(g[j] * s) * (u[j] * s);
      if (valid) {
        const size_t off = static_cast<size_t>(tok) * a.inter + col0 / 2 + 32 * c;
        if (a.act_f32)
          st_f32x32(a.act_f32 + off, g);
        else
          st_bf16x32(a.act + off, g);
      }
    }
    return;
  }
  // kModeQKV: a 32-column chunk never straddles a head or a q/k/v section (D >= 32)
  const int qdim = a.n_q * D, kvdim = a.n_kv * D;
  const int b = tok / a.seq_len, p = tok - b * a.seq_len;
  const int pos = a.pos_offset + p;
  const int half = D >> 1;
  // (cos, sin) of frequency d at this token's position: column `pos` of the dimension-major table,
  // so the warp's 32 consecutive tokens read one frequency as contiguous memory
  const float2* cs_col = a.rope_t + pos;
  auto dst_of = [&](int col) -> __nv_bfloat16* {
    if (col < qdim) return a.q_out + static_cast<size_t>(tok) * qdim + col;
    const int sec = col < qdim + kvdim ? 1 : 2;
    const int c2 = col - qdim - (sec == 2 ? kvdim : 0);
    const int kvh = c2 / D, d = c2 - kvh * D;
    __nv_bfloat16* base = sec == 1 ? a.k_out : a.v_out;
    return base + ((static_cast<size_t>(b) * a.n_kv + kvh) * a.kv_seq + p) * D + d;
  };
  const int cph = D >> 5;   // 32-column chunks per head
  // trace (first epilogue thread, SM cycles): 10 first 128-column group entered, 11 its first head's
  // RMS pass done, 12 that head's RoPE pass done, 13 the tile's second group done
  const bool cmk = a.trace && threadIdx.x == 64;
  const int grp = (col0 >> 7) & 1;
  auto cmark = [&](int slot) {
    if (cmk) const_cast<unsigned long long*>(a.trace)[blockIdx.x * kGemmTraceSlots + slot] = clock64();
  };
  if (grp == 0) cmark(10);
#pragma unroll 1
  for (int h0 = 0; h0 < 4; h0 += cph) {
    const int colh = col0 + 32 * h0;
    const bool is_v = colh >= qdim + kvdim;
    if (is_v) {
#pragma unroll 1
      for (int c = h0; c < h0 + cph; ++c) {
        float v[32];
        ld(c, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= s;
        if (valid) st_bf16x32(dst_of(col0 + 32 * c), v);
      }
      continue;
    }
    const float* gain = sgain ? (colh < qdim ? sgain : sgain + D) : (colh < qdim ? a.q_gain : a.k_gain);
    // the (cos, sin) of the first RoPE chunk's 32 dimensions, requested before the RMS pass so their
    // latency overlaps its TMEM loads; each later chunk's are requested while the previous one is stored
    float2 cs[32];
    if (D > 32) {
#pragma unroll
      for (int j = 0; j < 32; ++j) cs[j] = cs_col[static_cast<size_t>(j) * a.rope_ld];
    }
    // pass 1: RMS of the head
    float ss = 0.f;
#pragma unroll 1
    for (int c = h0; c < h0 + cph; ++c) {
      float v[32];
      ld(c, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) ss += v[j] * v[j];
    }
    const float rn = s * rsqrtf(ss * s * s / D + a.eps);
    if (grp == 0 && h0 == 0) cmark(11);
    if (D == 32) {
      // one chunk, pairs (j, j + 16)
      float v[32];
      ld(h0, v);
      float o[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float x0 = v[j] * rn * gain[j], x1 = v[j + 16] * rn * gain[j + 16];
        const float2 cs = cs_col[static_cast<size_t>(j) * a.rope_ld];
        o[j] = x0 * cs.x - x1 * cs.y;
        o[j + 16] = x1 * cs.x + x0 * cs.y;
      }
      if (valid) st_bf16x32(dst_of(colh), o);
    } else {
      // chunk c (head dims 32c'..) pairs with chunk c + cph/2
#pragma unroll 1
      for (int c = 0; c < cph / 2; ++c) {
        float lo[32], hi[32];
        ld(h0 + c, lo);
        ld(h0 + c + cph / 2, hi);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int d = 32 * c + jj;
          const float x0 = lo[jj] * rn * gain[d], x1 = hi[jj] * rn * gain[d + half];
          lo[jj] = x0 * cs[jj].x - x1 * cs[jj].y;
          hi[jj] = x1 * cs[jj].x + x0 * cs[jj].y;
        }
        if (c + 1 < cph / 2) {
#pragma unroll
          for (int j = 0; j < 32; ++j) cs[j] = cs_col[static_cast<size_t>(32 * (c + 1) + j) * a.rope_ld];
        }
        if (valid) {
          st_bf16x32(dst_of(colh + 32 * c), lo);
          st_bf16x32(dst_of(colh + 32 * c + half), hi);
        }
      }
    }
    if (grp == 0 && h0 == 0) cmark(12);
  }
  if (grp == 1) cmark(13);
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 2)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmArgs a) {
  using L = GemmSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kPipe);
  uint64_t* empty = full + STAGES;
  uint64_t* tmem_full = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* last_flag = reinterpret_cast<int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x, n_tile = blockIdx.y, split = blockIdx.z;
  const int KB = (a.K + 63) >> 6;
  const int kb0 = split * a.kb_per_split;
  const int kb1 = min(KB, kb0 + a.kb_per_split);
  const int nkb = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0 && nkb > 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const CUtensorMap* wmap = a.swap ? &tmA : &tmB;
      const CUtensorMap* xmap = a.swap ? &tmB : &tmA;
      const int wrow = a.swap ? m_tile * 128 : n_tile * BN;
      const int xrow = a.swap ? n_tile * BN : m_tile * 128;
      auto wdst = [&](int s) { return smem + s * L::kStage + (a.swap ? 0 : L::kA); };
      auto xdst = [&](int s) { return smem + s * L::kStage + (a.swap ? L::kA : 0); };
      const int pre = nkb < STAGES ? nkb : STAGES;
      // model weights do not depend on the previous kernel: request them before the dependency wait
      if (!a.w_stable) pdl_wait();
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], L::kStage);
        tma_load_2d(wdst(i), wmap, &full[i], (kb0 + i) * 64, wrow, pol_w);
      }
      if (a.w_stable) pdl_wait();
      for (int i = 0; i < pre; ++i) tma_load_2d(xdst(i), xmap, &full[i], (kb0 + i) * 64, xrow, pol_x);
      int last_issued = pre - 1;
      for (int i = pre; i < nkb; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&empty[s], ((i / STAGES) - 1) & 1, abort_flag)) {
          *abort_flag = 1;
          raise_error(a.err, kErrTimeoutProducer);
          break;
        }
        mbar_arrive_expect_tx(&full[s], L::kStage);
        tma_load_2d(wdst(s), wmap, &full[s], (kb0 + i) * 64, wrow, pol_w);
        tma_load_2d(xdst(s), xmap, &full[s], (kb0 + i) * 64, xrow, pol_x);
        last_issued = i;
      }
      // every copy must have landed before the CTA's shared memory is released
      // (immediate in the normal case: the MMA warp consumed them all)
      for (int i = last_issued - STAGES + 1; i <= last_issued; ++i) {
        if (i < 0) continue;
        if (!mbar_wait(&full[i % STAGES], (i / STAGES) & 1, nullptr, kDrainTimeoutNs))
          raise_error(a.err, kErrDrain);
      }
    } else if (lane == 0) {
      pdl_wait();
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, BN);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&full[s], (i / STAGES) & 1, abort_flag)) {
          *abort_flag = 1;
          raise_error(a.err, kErrTimeoutMma);
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * L::kStage);
        const uint32_t b_addr = a_addr + L::kA;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem, sw128_kmajor_desc(a_addr + 32 * k), sw128_kmajor_desc(b_addr + 32 * k), idesc,
                    (i | k) != 0 ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(tmem_full);
      // every MMA must be complete before TMEM is released
      if (!mbar_wait(tmem_full, 0, nullptr, kWaitTimeoutNs + kDrainTimeoutNs)) raise_error(a.err, kErrDrain);
    }
  } else {
    // ------------------------------------------------ epilogue warps 2..5
    const int wid = warp - 2;
    const int lane_base = (warp & 3) * 32;   // TMEM lanes this warp may read
    pdl_wait();
    const bool ok = mbar_wait(tmem_full, 0, abort_flag);
    if (!ok) {
      *abort_flag = 1;
      raise_error(a.err, kErrTimeoutEpilogue);
    }
    named_bar_sync(1, 128);
    // read once after the barrier: no role raises the flag after the accumulator is committed,
    // so all four warps take the same branch below
    const bool go = *abort_flag == 0;
    if (go) {
      tc_fence_after();
      const uint32_t tl = tmem + (static_cast<uint32_t>(lane_base) << 16);
      if (!a.swap) {
        // TMEM lane = token row of this tile
        const int tok = m_tile * 128 + lane_base + lane;
        const bool valid = tok < a.M;
        if (BN >= 128) {
          for (int g = 0; g < BN / 128; ++g) {
            const uint32_t tg = tl + g * 128;
            row_epilogue<false>(a, tok, valid, n_tile * BN + g * 128,
                                [&](int c, float (&v)[32]) { tmem_ld32(tg + c * 32, v); });
          }
        } else {   // 64-column tile: residual / store modes only
          row_epilogue<false>(a, tok, valid, n_tile * BN,
                              [&](int c, float (&v)[32]) { tmem_ld32(tl + c * 32, v); }, BN / 32);
        }
      } else {
        // lanes = output features, columns = tokens: add this split's partial sums
        const int feat = m_tile * 128 + lane_base + lane;
        float* dst = a.mode == kModeResid ? a.h : a.acc;
        const int ld = a.mode == kModeResid ? a.H : a.ld_acc;
        const int tokbase = n_tile * BN;
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld32(tl + c * 32, v);
          // residual with a gate: this split's partial of the gated sublayer output (linear in acc)
          const float gt = (a.mode == kModeResid && a.col_gate) ? a.col_gate[feat] : 1.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tok = tokbase + c * 32 + j;
            if (tok < a.tokens) atomicAdd(dst + static_cast<size_t>(tok) * ld + feat, v[j] * gt);
          }
        }
        __threadfence();
        named_bar_sync(1, 128);
        if (wid == 0 && lane == 0) {
          const int prev = atomicAdd(a.counters + m_tile, 1);
          const int last = prev == static_cast<int>(gridDim.z) - 1;
          if (last) a.counters[m_tile] = 0;
          *last_flag = last;
        }
        named_bar_sync(1, 128);
        if (*last_flag && a.mode != kModeStoreF32) {
          __threadfence();
          // the last CTA of this feature tile: one thread per token
          const int tok = wid * 32 + lane;
          const bool valid = tok < a.tokens;
          float* row = dst + static_cast<size_t>(valid ? tok : 0) * ld + m_tile * 128;
          const bool zero_after = a.mode != kModeResid;
            row_epilogue<true>(a, tok, valid, m_tile * 128, [&](int c, float (&v)[32]) {
            if (valid) {
              ld_f32x32(row + 32 * c, v);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = 0.f;
            }
          });
            if (zero_after && valid) {   // leave the split-K scratch zeroed for the next launch
            float4* r4 = reinterpret_cast<float4*>(row);
#pragma unroll
            for (int i = 0; i < 32; ++i) r4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace dm0

namespace dm0 {

// ---------------------------------------------------------------- persistent normal-orientation GEMM
//
// One CTA per SM walks output tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...
// in a banded raster: bands of band_m m-tiles, m fastest inside a band, so the
// CTAs running together cover a few weight tiles and at most band_m activation
// tiles (activation tiles are read from DRAM once if the band stays in L2,
// weights once per band).  band_m = 1 is the n-fastest raster: the CTAs of a
// wave share a few activation tiles and the whole weight matrix, which then
// has to stay in L2 for the whole launch (the host picks it when the weights
// are small next to L2; with tall bands the residual and output streams of the
// epilogues evict the band's activations).  The producer streams
// k-blocks of consecutive tiles through one ring without pausing between tiles,
// and the accumulator is double-buffered in TMEM (2 x BN columns): while the
// epilogue warps finish tile i from one buffer, the MMA warp already
// accumulates tile i+1 into the other.
constexpr int kBandM = 64;   // default m-tiles per raster band (band_m <= 0)

// output tile index t -> (m_tile, n_tile) in the banded raster
__device__ __forceinline__ void band_tile(int t, int mt, int nt, int band_m, int& m_tile, int& n_tile) {
  const int bh = band_m > 0 ? band_m : kBandM;
  const int band = t / (bh * nt);
  const int m0 = band * bh;
  const int bm = min(bh, mt - m0);   // m-tiles in this band
  const int r = t - band * bh * nt;
  m_tile = m0 + r % bm;
  n_tile = r / bm;
}

template <int BN, int STAGES, int EPI = 8>
struct PGemmSmem {
  static constexpr uint32_t kA = 128 * 128;
  static constexpr uint32_t kB = BN * 128;
  static constexpr uint32_t kStage = kA + kB;
  static constexpr uint32_t kPipe = STAGES * kStage;
  static constexpr uint32_t kOffScr = kPipe + 256;            // after the barriers
  static constexpr uint32_t kScrWarp = ResidScratch::kBytes;  // per epilogue warp
  static constexpr uint32_t kBytes = kOffScr + EPI * kScrWarp + 1024;
  static constexpr uint32_t kTmemCols = 2 * BN;
  static_assert(kBytes <= 232448, "shared memory per CTA");
};

// kF8: both operands FP8 E4M3 (tensor maps of bytes), a k-block is 128 values instead of 64 (the
// same 128-byte rows, so the ring, the swizzle and the descriptors are unchanged), and the epilogue
// applies the per-token and per-output-channel scales.
template <int BN, int STAGES, bool kF8 = false, int EPI = 8>
__global__ void __launch_bounds__(PGemmWarps<EPI>::kThreads, 1)
    gemm_tc_persistent(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const GemmArgs a) {
  using L = PGemmSmem<BN, STAGES, EPI>;
  constexpr int kKB = kF8 ? 128 : 64;   // operand values per 128-byte k-block row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kPipe);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;   // [2] accumulator buffer complete
  uint64_t* tempty = tfull + 2;       // [2] epilogue finished with the buffer
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = (a.K + kKB - 1) / kKB;
  const int mt = (a.M + 127) >> 7;
  const int ntiles = mt * (a.N / BN);

  if (threadIdx.x == 0) {
    if (a.trace)   // this CTA's row: clear the marks a previous launch may have left
      for (int i = 0; i < kGemmTraceSlots - 2; ++i) a.trace[blockIdx.x * kGemmTraceSlots + i] = 0ull;
    gemm_mark(a.trace, kGtEntry);
    if (a.trace && blockIdx.x == 0) {
      a.trace[kGemmTraceSlots - 2] = (static_cast<unsigned long long>(a.M) << 32) | static_cast<unsigned>(a.N);
      a.trace[kGemmTraceSlots - 1] = (static_cast<unsigned long long>(a.K) << 32) | static_cast<unsigned>(BN);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], EPI);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  // QKV: the QK-norm gains (weights, which no kernel writes) staged once per launch in the epilogue
  // scratch, which only the residual mode uses otherwise
  float* sgain = a.mode == kModeQKV && a.q_gain && a.k_gain && 8 * a.head_dim <= static_cast<int>(EPI * L::kScrWarp)
                     ? reinterpret_cast<float*>(smem + L::kOffScr)
                     : nullptr;
  if (sgain)
    for (int i = threadIdx.x; i < 2 * a.head_dim; i += blockDim.x)
      sgain[i] = i < a.head_dim ? a.q_gain[i] : a.k_gain[i - a.head_dim];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  if (threadIdx.x == 0) gemm_mark(a.trace, kGtSetup);

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      const uint64_t pol_w = policy_evict_last();   // a weight tile is shared by the CTAs running together
      const uint64_t pol_x = policy_evict_first();
      int it = 0;
      bool waited = false;
      // the first tile's weight k-blocks may be requested before the dependency wait
      const int first = blockIdx.x;
      int pre = 0;
      if (a.w_stable && first < ntiles) {
        pre = KB < STAGES ? KB : STAGES;
        int m_first, n0;
        band_tile(first, mt, a.N / BN, a.band_m, m_first, n0);
        for (int k = 0; k < pre; ++k) {
          mbar_arrive_expect_tx(&full[k], L::kStage);
          tma_load_2d(smem + k * L::kStage + L::kA, &tmB, &full[k], k * kKB, n0 * BN, pol_w);
        }
      }
      pdl_wait();
      waited = true;
      (void)waited;
      gemm_mark(a.trace, kGtDepWait);
      for (int t = first; t < ntiles && !*abort_flag; t += gridDim.x) {
        int mtile, ntile;
        band_tile(t, mt, a.N / BN, a.band_m, mtile, ntile);
        const int m0 = mtile * 128, n0 = ntile * BN;
        for (int k = 0; k < KB; ++k, ++it) {
          const int s = it % STAGES;
          if (it < pre) {   // weight half already requested
            tma_load_2d(smem + s * L::kStage, &tmA, &full[s], k * kKB, m0, pol_x);
            continue;
          }
          if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) - 1) & 1, abort_flag)) {
            *abort_flag = 1;
            raise_error(a.err, kErrTimeoutProducer);
            break;
          }
          mbar_arrive_expect_tx(&full[s], L::kStage);
          tma_load_2d(smem + s * L::kStage, &tmA, &full[s], k * kKB, m0, pol_x);
          tma_load_2d(smem + s * L::kStage + L::kA, &tmB, &full[s], k * kKB, n0, pol_w);
        }
      }
      gemm_mark(a.trace, kGtLastLoad);
      for (int i = it - STAGES; i < it; ++i) {   // copies in flight land before the CTA exits
        if (i < 0) continue;
        if (!mbar_wait(&full[i % STAGES], (i / STAGES) & 1, nullptr, kDrainTimeoutNs)) raise_error(a.err, kErrDrain);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = kF8 ? idesc_e4m3_f32(128, BN) : idesc_bf16_f32(128, BN);
      int it = 0, local = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++local) {
        const int buf = local & 1;
        if (local >= 2 && !mbar_wait(&tempty[buf], ((local >> 1) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int k = 0; k < KB; ++k, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, abort_flag)) {
            ok = false;
            break;
          }
          if (it == 0) gemm_mark(a.trace, kGtFirstStage);
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * L::kStage);
          const uint32_t b_addr = a_addr + L::kA;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            if constexpr (kF8)
              umma_e4m3(tmem + buf * BN, sw128_kmajor_desc(a_addr + 32 * kk), sw128_kmajor_desc(b_addr + 32 * kk),
                        idesc, (k | kk) != 0 ? 1u : 0u);
            else
              umma_bf16(tmem + buf * BN, sw128_kmajor_desc(a_addr + 32 * kk), sw128_kmajor_desc(b_addr + 32 * kk),
                        idesc, (k | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (local == 0) gemm_mark(a.trace, kGtFirstIssued);
        if (ok) umma_commit(&tfull[buf]);
      }
      if (!ok) {
        *abort_flag = 1;
        raise_error(a.err, kErrTimeoutMma);
      }
      umma_commit(drain);
      if (!mbar_wait(drain, 0, nullptr, kWaitTimeoutNs + kDrainTimeoutNs)) raise_error(a.err, kErrDrain);
    }
  } else {
    // epilogue warps 2..9: lane quarter (warp mod 4) and column half hf.  A 256-wide tile's two
    // 128-column groups go one to each half; a 128-wide tile of the column-independent modes
    // (residual, store) splits into two 64-column halves, the QKV and SwiGLU groups stay whole (half 0);
    // a 64-wide tile is half 0's
    const int lane_base = (warp & 3) * 32;
    const int hf = (warp - 2) >> 2;
    pdl_wait();
    // residual epilogue: the rows of the CTA's next tile are requested into L2 one tile ahead, so the
    // h loads of that tile hit L2 while the accumulator of the current tile drains
    auto prefetch_rows = [&](int t) {
      if (a.mode != kModeResid || t >= ntiles || hf != 0) return;
      int m_tile, n_tile;
      band_tile(t, mt, a.N / BN, a.band_m, m_tile, n_tile);
      const int tok = m_tile * 128 + lane_base + lane;
      if (tok < a.M) prefetch_l2_bulk(a.h + static_cast<size_t>(tok) * a.H + n_tile * BN, BN * 4);
    };
    prefetch_rows(blockIdx.x);
    const bool col_indep = a.mode == kModeResid || a.mode == kModeStoreF32;
    int local = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
      const int buf = local & 1;
      if (!mbar_wait(&tfull[buf], (local >> 1) & 1, abort_flag)) {
        *abort_flag = 1;
        raise_error(a.err, kErrTimeoutEpilogue);
        break;
      }
      if (local == 0 && threadIdx.x == 64) gemm_mark(a.trace, kGtFirstAcc);
      tc_fence_after();
      prefetch_rows(t + gridDim.x);
      int m_tile, n_tile;
      band_tile(t, mt, a.N / BN, a.band_m, m_tile, n_tile);
      const uint32_t tl = tmem + (static_cast<uint32_t>(lane_base) << 16) + buf * BN;
      const int tok = m_tile * 128 + lane_base + lane;
      const bool valid = tok < a.M;
      // FP8: the token's activation scale (0 for rows past M, whose stores are predicated off anyway)
      const float rs = kF8 && valid ? __ldg(a.row_scale + tok) : 0.f;
      auto scaled = [&](uint32_t taddr, int col, float (&v)[32]) {
        tmem_ld32(taddr, v);
        if constexpr (kF8) {
          const float4* cs4 = reinterpret_cast<const float4*>(a.col_scale + col);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 cs = __ldg(cs4 + i);
            v[4 * i] *= rs * cs.x;
            v[4 * i + 1] *= rs * cs.y;
            v[4 * i + 2] *= rs * cs.z;
            v[4 * i + 3] *= rs * cs.w;
          }
        }
      };
      // this warp's columns of the tile: [c0, c0 + 32 nch) relative to the tile
      int c0 = 0, nch = 0;
      if (EPI == 4) {   // one warp per lane quarter walks the whole tile, 128-column group by group
        for (int g = 0; g < (BN >= 128 ? BN / 128 : 1); ++g) {
          const uint32_t tg = tl + g * 128;
          const int col0 = n_tile * BN + g * 128;
          const int ng = BN >= 128 ? 4 : BN / 32;
          if (a.mode == kModeResid) {
            uint8_t* scr = smem + L::kOffScr + (warp - 2) * L::kScrWarp;
            resid_epilogue_warp(a, m_tile * 128 + lane_base, col0, ng, scr,
                                [&](int c, float (&v)[32]) { scaled(tg + c * 32, col0 + 32 * c, v); });
          } else {
            row_epilogue<false>(a, tok, valid, col0,
                                [&](int c, float (&v)[32]) { scaled(tg + c * 32, col0 + 32 * c, v); }, ng, sgain);
          }
        }
      } else if (BN == 256) {
        c0 = 128 * hf;
        nch = 4;
      } else if (BN == 128) {
        c0 = col_indep ? 64 * hf : 0;
        nch = col_indep ? 2 : (hf == 0 ? 4 : 0);
      } else {
        nch = hf == 0 ? BN / 32 : 0;
      }
      if (nch > 0) {
        const uint32_t tg = tl + c0;
        const int col0 = n_tile * BN + c0;
        if (a.mode == kModeResid) {
          uint8_t* scr = smem + L::kOffScr + (warp - 2) * L::kScrWarp;
          resid_epilogue_warp(a, m_tile * 128 + lane_base, col0, nch, scr,
                              [&](int c, float (&v)[32]) { scaled(tg + c * 32, col0 + 32 * c, v); });
        } else {
          row_epilogue<false>(a, tok, valid, col0,
                              [&](int c, float (&v)[32]) { scaled(tg + c * 32, col0 + 32 * c, v); }, nch, sgain);
        }
      }
      // the accumulator buffer is free for tile local + 2
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (threadIdx.x == 64) gemm_mark(a.trace, local == 0 ? kGtFirstDone : kGtLastDone);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) gemm_mark(a.trace, kGtExit);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace dm0
