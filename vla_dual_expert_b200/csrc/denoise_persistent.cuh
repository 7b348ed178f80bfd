// The whole Euler loop of a single observation (DM0.5 page, sections 5.2-5.3:
// K steps of x <- x + dt v(x, t) over the 50 x 32 action chunk, each velocity
// a pass of the 28 action-expert layers over [prefix cache; suffix]) as ONE
// persistent kernel: one CTA per SM, and a grid-wide barrier where the next
// phase needs a whole tensor that other CTAs produced.
//
// Why: at one observation every GEMM streams a weight matrix of 4-13 MB
// against 50 tokens, so a kernel per GEMM is a chain of launch, prologue,
// first-load and split-K latencies (~15-30 us each, ~140 per step) rather than
// a weight stream.  Here weights do not depend on activations, so the TMA
// producer warp of every CTA runs ahead across phase and layer boundaries,
// limited only by its shared-memory ring; the dependent chain per phase is one
// grid barrier, one L2 round trip to stage the activation operand, the MMAs
// and the fp32 reductions.
//
// Per layer l, five phases (T = tokens <= 64, the padded MMA N is 64):
//   A  qkv_acc[t][f]  += sum_k Wqkv[f][k] * bf16(g_attn[k] h[t][k])   split-K over all CTAs
//                       (tile-0 CTAs also add sum_k h[t][k]^2 for the pending RMSNorm)
//   B  attention: one CTA per (KV head, key split).  The CTA finishes q of
//      its G query heads (1/rms, QK-RMSNorm, RoPE at position P + t) and, if it
//      owns the suffix block, the suffix K/V, then runs 64-key blocks of the
//      prefix cache (TMA) and the suffix (shared memory) through tcgen05:
//      S = Q K^T and O += P V in TMEM; it stores its partial O / l in bf16
//      with its (max, sum).
//   C  h[t][f] += sum_k Wo[f][k] * o[t][k], the B operand o combined from the
//      key splits while it is staged (residual add by fp32 reduction into h)
//   D  gu_acc[t][f] += sum_k Wgu[f][k] * bf16(g_mlp[k] h[t][k])  (+ MLP sum of squares)
//   E  h[t][f] += sum_k Wd[f][k] * bf16(silu(gate / rms) * (up / rms))
// and after layer L-1 the step boundary (velocity, Euler update, next input;
// one CTA per token).  The GEMM work of a phase, (128-row weight tile, 64-wide
// k-block) pairs in tile-major order, is cut into contiguous equal ranges, one
// per CTA; a range covers at most two tiles, each accumulated in its own
// 64-column TMEM segment.
//
// Warp roles (320 threads): warp 0 TMA producer (weights, prefix K/V), warp 1
// TMEM owner and tcgen05.mma issuer, warps 2-9 everything else: operand
// staging (every thread issues all of its L2 loads before using any, so a
// stage costs one round trip), reductions (two warps per TMEM lane quarter,
// one per 32-column half), grid barriers; warps 2-5 also run the softmax.
// Every wait is bounded; a CTA that gives up raises the device error word and
// a global abort word that every other CTA's barrier polls, so the whole grid
// unwinds.
#pragma once
#include "attention_tc.cuh"
#include "elementwise.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace dm0 {

#ifndef DM0_PD_COMPUTE_WARPS
#define DM0_PD_COMPUTE_WARPS 8
#endif
constexpr int kPdCompute = 32 * DM0_PD_COMPUTE_WARPS;   // warps 2.. (4 or 8)
constexpr int kPdThreads = 64 + kPdCompute;
constexpr int kPdHalves = kPdCompute / 128;              // warps sharing a TMEM lane quarter
constexpr int kPdStages = 4;       // 16 KB ring stages
constexpr int kPdBTiles = 6;       // staged activation tiles per GEMM phase
constexpr int kPdMaxSplits = 8;    // attention key splits per KV head
// trace marks per (phase, CTA): 0 phase start, 1 operand staged, 2 first accumulator / S tile
// ready, 3 results issued, 4 after the release fence, 5 barrier arrival, 6 MMA warp saw the
// operand, 7 MMA warp issued its last MMA of the phase
// 8 operand copies issued, 9 copies landed; attention: 10 / 12 S of block 0 / 1 read, 11 / 13 P of
// block 0 / 1 written, 14 O readout, 15 MMA warp issued PV of block 0
constexpr int kPdTraceSlots = 16;

struct PdSmem {
  static constexpr uint32_t kStage = 16384;                 // 128 weight rows x 64 k, or 64 keys x 128 dims
  static constexpr uint32_t kOffRing = 0;
  static constexpr uint32_t kOffWork = kPdStages * kStage;
  // GEMM phases: B tiles, then gain rows / sums of squares, then the landing area of the operand copies
  static constexpr uint32_t kBTile = 8192;                  // 64 tokens x 64 k
  static constexpr uint32_t kOffAux = kOffWork + kPdBTiles * kBTile;   // 2 KB
  static constexpr uint32_t kOffLandG = kOffAux + 2048;
  // attention phase: Q, P[2], suffix K, V, then the landing area of the q / k / v rows
  static constexpr uint32_t kOffQ = kOffWork;               // 128 rows x 128 dims (two SW128 halves)
  static constexpr uint32_t kOffP = kOffQ + 32768;          // 2 x (128 rows x 64 keys)
  static constexpr uint32_t kOffSK = kOffP + 32768;         // 64 keys x 128 dims (two 8 KB halves)
  static constexpr uint32_t kOffSV = kOffSK + 16384;
  static constexpr uint32_t kOffLandA = kOffSV + 16384;     // 128 rows x 128 fp32
  static constexpr uint32_t kWork = 163840;
  static constexpr uint32_t kOffBar = kOffWork + kWork;     // barriers, then sx[64], sred[8]
  static constexpr uint32_t kOffMisc = kOffBar + 512;
  static constexpr uint32_t kSlack = 1024;
  static constexpr uint32_t kBytes = kOffBar + 1024 + kSlack;
  static constexpr uint32_t kLandG = kOffWork + kWork - kOffLandG;   // bytes
  static_assert(kOffLandA + 65536 <= kOffWork + kWork, "attention landing area overflows the work area");
};

struct PdLayer {
  const float *attn_norm, *q_norm, *k_norm, *mlp_norm;
};

struct PdArgs {
  int L, T, P, steps;       // layers, tokens (<= 64), prefix length, Euler steps
  int Ha, Ia, n_q, n_kv;    // head_dim is 128
  int QR;                   // (n_q + 2 n_kv) * 128
  float eps, scale_log2;
  int splits, bps;          // attention: key splits per KV head, 64-key blocks per split
  const PdLayer* layers;    // [L]
  const float2* rope;       // [position][64] (cos, sin)
  float* h;                 // [T][Ha] residual stream
  float* acc_qkv;           // [T][QR]  zero at launch
  float* acc_gu;            // [T][2 Ia]
  float* ssq;               // [2][T]: attention-norm and MLP-norm sums of squares, zero at launch
  __nv_bfloat16* part_o;    // [n_kv * splits][128 rows][128]: O / l of the split
  float2* part_ml;          // [n_kv * splits][128 rows]: (max, sum) of the split
  unsigned* sync;           // [0] barrier arrivals, [1] abort; zero at launch
  int* err;
  unsigned long long* trace;  // optional [phase][CTA][kPdTraceSlots] %globaltimer marks; null: off
  StepArgs step;            // x, h, W_in, b_in, final_norm, W_out, b_out, Ha, A, eps, steps, tokens, vel
};

__device__ __forceinline__ void pd_geom(const PdArgs& a, int ph, int& tiles, int& nkb, int& rows_pl) {
  if (ph == 0) {
    tiles = a.QR >> 7, nkb = a.Ha >> 6, rows_pl = a.QR;
  } else if (ph == 2) {
    tiles = a.Ha >> 7, nkb = a.n_q * 2, rows_pl = a.Ha;
  } else if (ph == 3) {
    tiles = a.Ia >> 6, nkb = a.Ha >> 6, rows_pl = 2 * a.Ia;
  } else {
    tiles = a.Ha >> 7, nkb = a.Ia >> 6, rows_pl = a.Ha;
  }
}
__device__ __forceinline__ void pd_range(int total, int c, int n, int& p0, int& p1) {
  p0 = static_cast<int>(static_cast<long long>(total) * c / n);
  p1 = static_cast<int>(static_cast<long long>(total) * (c + 1) / n);
}
// byte offset of 16-byte chunk c16 of row `row` in a SW128 K-major tile (128-byte rows, 1024-aligned base)
__device__ __forceinline__ uint32_t sw_chunk(int row, int c16) {
  return static_cast<uint32_t>(row * 128 + ((c16 ^ (row & 7)) << 4));
}
__device__ __forceinline__ uint4 pack8(const float* v) {
  return make_uint4(bf2(v[0], v[1]), bf2(v[2], v[3]), bf2(v[4], v[5]), bf2(v[6], v[7]));
}
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Operand staging, one function per phase type, kept out of line.  Every compute thread first
// issues 16-byte cp.async copies of its share of the phase's L2 data into a shared-memory landing
// area (no registers are held while the copies are in flight, so the whole stage costs one L2 round
// trip), then the operand is built from shared memory.  A unit of the build is one 16-byte bf16
// chunk (8 values) of a staged row; unit u goes to compute thread u % kPdCompute, so the 8 chunks of
// a 64-column row segment sit in 8 adjacent lanes and a thread keeps the chunk index c8 = ct % 8.
__device__ __forceinline__ void pd_cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// commit this thread's copies and wait for all of them
__device__ __forceinline__ void pd_cp_wait() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// (A, D) bf16(g * h) for pairs [p0, p0 + np); weight tile 0 also adds sum h^2 into ssq
template <int kT>
__device__ __noinline__ void pd_stage_norm(const PdArgs& a, uint8_t* smem, int ct, int p0, int np, int nkb,
                                           const float* gain, float* ssq, unsigned long long* mk) {
  using SM = PdSmem;
  const int T = kT > 0 ? kT : a.T;   // tokens; a compile-time constant for the common shape
  const int c8 = ct & 7;
  float* land = reinterpret_cast<float*>(smem + SM::kOffLandG);   // [np][T][64]
  float* sg = reinterpret_cast<float*>(smem + SM::kOffAux);       // [np][64]
  const float* h = a.h;
  const int Ha = a.Ha;
  int kb = p0 % nkb;
  for (int i = 0; i < np; ++i) {
    for (int q = ct; q < T * 16; q += kPdCompute) {
      const int t = q >> 4, c = q & 15;
      pd_cp16(land + (i * T + t) * 64 + c * 4, h + static_cast<size_t>(t) * Ha + kb * 64 + c * 4);
    }
    if (ct < 16) pd_cp16(sg + i * 64 + ct * 4, gain + kb * 64 + ct * 4);
    if (++kb == nkb) kb = 0;
  }
  if (mk && ct == 0) mk[8] = globaltimer();
  pd_cp_wait();
  named_bar_sync(1, kPdCompute);
  if (mk && ct == 0) mk[9] = globaltimer();
  const int tile0_pairs = p0 < nkb ? min(np, nkb - p0) : 0;   // pairs of weight tile 0 add to ssq
  for (int i = 0; i < np; ++i) {
    for (int base = 0; base < T * 8; base += kPdCompute) {   // validity is uniform over each 8-lane group
      const int u = base + ct;
      const int t = u >> 3;
      float ss = 0.f;
      if (t < T) {
        const float4* x4 = reinterpret_cast<const float4*>(land + (i * T + t) * 64 + c8 * 8);
        const float4* g4 = reinterpret_cast<const float4*>(sg + i * 64 + c8 * 8);
        const float4 x0 = x4[0], x1 = x4[1], g0 = g4[0], g1 = g4[1];
        ss = x0.x * x0.x + x0.y * x0.y + x0.z * x0.z + x0.w * x0.w + x1.x * x1.x + x1.y * x1.y + x1.z * x1.z +
             x1.w * x1.w;
        const float y[8] = {g0.x * x0.x, g0.y * x0.y, g0.z * x0.z, g0.w * x0.w,
                            g1.x * x1.x, g1.y * x1.y, g1.z * x1.z, g1.w * x1.w};
        *reinterpret_cast<uint4*>(smem + SM::kOffWork + i * SM::kBTile + sw_chunk(t, c8)) = pack8(y);
      }
      if (i < tile0_pairs) {
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        ss += __shfl_xor_sync(0xffffffffu, ss, 4);
        if (t < T && c8 == 0) atomicAdd(ssq + t, ss);
      }
    }
  }
}

// (C) attention output o = sum_j w_j o_j / sum_j w_j, w_j = l_j 2^(m_j - max m), over the key splits
template <int kT>
__device__ __noinline__ void pd_stage_attn_out(const PdArgs& a, uint8_t* smem, int ct, int p0, int np, int nkb, unsigned long long* mk) {
  using SM = PdSmem;
  const int T = kT > 0 ? kT : a.T;   // tokens; a compile-time constant for the common shape
  const int c8 = ct & 7;
  const int G = a.n_q / a.n_kv, S = a.splits;
  __nv_bfloat16* lo = reinterpret_cast<__nv_bfloat16*>(smem + SM::kOffLandG);   // [np][S][T][64]
  float2* lml = reinterpret_cast<float2*>(lo + static_cast<size_t>(np) * S * T * 64);   // [np][S][T]
  int kb = p0 % nkb;
  for (int i = 0; i < np; ++i) {
    const int hq = kb >> 1, g2 = hq / G, hh = hq - g2 * G;
    for (int sp = 0; sp < S; ++sp) {
      const size_t src = (static_cast<size_t>(g2) * S + sp) * 128 + hh * T;   // row of token 0
      const int dst = (i * S + sp) * T;
      for (int q = ct; q < T * 8; q += kPdCompute) {
        const int t = q >> 3, c = q & 7;
        pd_cp16(lo + (dst + t) * 64 + c * 8, a.part_o + (src + t) * 128 + (kb & 1) * 64 + c * 8);
      }
      if ((src & 1) == 0 && (T & 1) == 0) {   // (m, l) of two tokens per 16-byte copy
        for (int q = ct; q < T / 2; q += kPdCompute) pd_cp16(lml + dst + 2 * q, a.part_ml + src + 2 * q);
      } else {
        for (int q = ct; q < T; q += kPdCompute) lml[dst + q] = __ldcg(a.part_ml + src + q);
      }
    }
    if (++kb == nkb) kb = 0;
  }
  if (mk && ct == 0) mk[8] = globaltimer();
  pd_cp_wait();
  named_bar_sync(1, kPdCompute);
  if (mk && ct == 0) mk[9] = globaltimer();
  for (int i = 0; i < np; ++i) {
    for (int u = ct; u < T * 8; u += kPdCompute) {
      const int t = u >> 3;
      float mx = -__int_as_float(0x7f800000);
      for (int sp = 0; sp < S; ++sp) mx = fmaxf(mx, lml[(i * S + sp) * T + t].x);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float den = 0.f;
      for (int sp = 0; sp < S; ++sp) {
        const float2 ml = lml[(i * S + sp) * T + t];
        const float w = ml.y * exp2f(ml.x - mx);
        den += w;
        const uint4 ov = *reinterpret_cast<const uint4*>(lo + ((i * S + sp) * T + t) * 64 + c8 * 8);
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(o2[e]);
          acc[2 * e] += w * f.x;
          acc[2 * e + 1] += w * f.y;
        }
      }
      const float inv = 1.f / den;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] *= inv;
      *reinterpret_cast<uint4*>(smem + SM::kOffWork + i * SM::kBTile + sw_chunk(t, c8)) = pack8(acc);
    }
  }
}

// (E) SwiGLU of the gate/up sums with 1/rms of the MLP norm
template <int kT>
__device__ __noinline__ void pd_stage_swiglu(const PdArgs& a, uint8_t* smem, int ct, int p0, int np, int nkb, unsigned long long* mk) {
  using SM = PdSmem;
  const int T = kT > 0 ? kT : a.T;   // tokens; a compile-time constant for the common shape
  const int c8 = ct & 7;
  const float inv_Ha = 1.0f / a.Ha;
  float* land = reinterpret_cast<float*>(smem + SM::kOffLandG);   // [np][T][128]: gate 64 | up 64
  float* sq = reinterpret_cast<float*>(smem + SM::kOffAux);       // [2T] both sums of squares
  const float* gu = a.acc_gu;
  const int ld = 2 * a.Ia;
  int kb = p0 % nkb;
  for (int i = 0; i < np; ++i) {
    for (int q = ct; q < T * 32; q += kPdCompute) {
      const int t = q >> 5, c = q & 31;
      pd_cp16(land + (i * T + t) * 128 + c * 4, gu + static_cast<size_t>(t) * ld + 128 * kb + c * 4);
    }
    if (++kb == nkb) kb = 0;
  }
  for (int q = T / 4 + ct; q < (2 * T + 3) / 4; q += kPdCompute) pd_cp16(sq + 4 * q, a.ssq + 4 * q);
  if (mk && ct == 0) mk[8] = globaltimer();
  pd_cp_wait();
  named_bar_sync(1, kPdCompute);
  if (mk && ct == 0) mk[9] = globaltimer();
  for (int i = 0; i < np; ++i) {
    for (int u = ct; u < T * 8; u += kPdCompute) {
      const int t = u >> 3;
      const float s = rsqrtf(sq[T + t] * inv_Ha + a.eps);
      const float4* g4 = reinterpret_cast<const float4*>(land + (i * T + t) * 128 + c8 * 8);
      const float4 ga = g4[0], gb = g4[1], ua = g4[16], ub = g4[17];
      const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
      const float uu[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = silu_f(gg[e] * s) * (uu[e] * s);
      *reinterpret_cast<uint4*>(smem + SM::kOffWork + i * SM::kBTile + sw_chunk(t, c8)) = pack8(y);
    }
  }
}

// Q rows (then the suffix K and V rows) of one attention item.  Build unit = (row, c8): dims
// [8 c8, 8 c8 + 8) and their RoPE partners [64 + 8 c8, ...) sit in one thread; a row's 8 units are
// adjacent lanes, so the head's sum of squares is a 3-step shuffle.
template <int kT>
__device__ __noinline__ void pd_stage_qkv(const PdArgs& a, uint8_t* smem, int ct, int l, int kvg, bool has_sfx, unsigned long long* mk) {
  using SM = PdSmem;
  const int T = kT > 0 ? kT : a.T;   // tokens; a compile-time constant for the common shape
  const int c8 = ct & 7;
  const int G = a.n_q / a.n_kv, GT = G * T;
  const int qd = a.n_q * 128, kvd = a.n_kv * 128;
  const float inv_Ha = 1.0f / a.Ha;
  const int QR = a.QR;
  const float* acc = a.acc_qkv;
  float* land = reinterpret_cast<float*>(smem + SM::kOffLandA);   // [128 rows][128]
  // the P buffers are idle while the operands are built: sums of squares, QK-norm gains, RoPE rows
  float* sq = reinterpret_cast<float*>(smem + SM::kOffP);             // [T]
  float* sgq = reinterpret_cast<float*>(smem + SM::kOffP + 256);      // [128]
  float* sgk = reinterpret_cast<float*>(smem + SM::kOffP + 768);      // [128]
  float2* srope = reinterpret_cast<float2*>(smem + SM::kOffP + 1280); // [T][64] (cos, sin) at P + t
  for (int set = 0; set < (has_sfx ? 2 : 1); ++set) {
    const bool kv = set == 1;
    // rows: Q (set 0) r < GT = (head-in-group r / T, token r % T); K (set 1) r < 64, V r >= 64
    if (!kv) {
      for (int r = 0; r < G; ++r)   // head r of the group: rows r T .. r T + T - 1
        for (int q = ct; q < T * 32; q += kPdCompute) {
          const int t = q >> 5, c = q & 31;
          pd_cp16(land + (r * T + t) * 128 + c * 4, acc + static_cast<size_t>(t) * QR + (kvg * G + r) * 128 + c * 4);
        }
      const PdLayer& ly = a.layers[l];
      for (int q = ct; q < (T + 3) / 4; q += kPdCompute) pd_cp16(sq + 4 * q, a.ssq + 4 * q);
      if (ct < 32) pd_cp16(sgq + 4 * ct, ly.q_norm + 4 * ct);
      else if (ct < 64) pd_cp16(sgk + 4 * (ct - 32), ly.k_norm + 4 * (ct - 32));
      for (int q = ct; q < T * 32; q += kPdCompute)
        pd_cp16(reinterpret_cast<float*>(srope) + 4 * q, reinterpret_cast<const float*>(a.rope + static_cast<size_t>(a.P) * 64) + 4 * q);
    } else {
      for (int w = 0; w < 2; ++w)
        for (int q = ct; q < T * 32; q += kPdCompute) {
          const int t = q >> 5, c = q & 31;
          pd_cp16(land + (w * 64 + t) * 128 + c * 4, acc + static_cast<size_t>(t) * QR + qd + w * kvd + kvg * 128 + c * 4);
        }
    }
    if (mk && ct == 0 && set == 0) mk[8] = globaltimer();
    pd_cp_wait();
    named_bar_sync(1, kPdCompute);
    if (mk && ct == 0 && set == 0) mk[9] = globaltimer();
    for (int u = ct; u < 1024; u += kPdCompute) {   // 128 rows x 8 units; warp-uniform trip count
      const int r = u >> 3;
      const bool valid = kv ? (r & 63) < T : r < GT;
      const int which = kv ? (r >> 6) : 0;
      const int t = kv ? (r & 63) : (valid ? r % T : 0);
      float x[16];
      if (valid) {
        const float4* s4 = reinterpret_cast<const float4*>(land + r * 128);
        const float4 v0 = s4[2 * c8], v1 = s4[2 * c8 + 1], v2 = s4[16 + 2 * c8], v3 = s4[16 + 2 * c8 + 1];
        x[0] = v0.x, x[1] = v0.y, x[2] = v0.z, x[3] = v0.w, x[4] = v1.x, x[5] = v1.y, x[6] = v1.z, x[7] = v1.w;
        x[8] = v2.x, x[9] = v2.y, x[10] = v2.z, x[11] = v2.w, x[12] = v3.x, x[13] = v3.y, x[14] = v3.z, x[15] = v3.w;
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = 0.f;
      }
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) ss += x[e] * x[e];
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      ss += __shfl_xor_sync(0xffffffffu, ss, 4);
      uint8_t* dst;
      uint32_t hstride;
      int drow;
      if (!kv) {
        dst = smem + SM::kOffQ, hstride = 16384, drow = r;
      } else {
        dst = smem + (which ? SM::kOffSV : SM::kOffSK), hstride = 8192, drow = r & 63;
      }
      if (valid) {
        const float s = rsqrtf(sq[t] * inv_Ha + a.eps);
        if (kv && which == 1) {   // V: 1/rms only
#pragma unroll
          for (int e = 0; e < 16; ++e) x[e] *= s;
        } else {                  // Q / K: 1/rms, RMSNorm over the head, RoPE at position P + t
          const float* gain = kv ? sgk : sgq;
          const float rn = s * rsqrtf(ss * s * s / 128.f + a.eps);
          const float2* cs = srope + t * 64 + c8 * 8;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int d = c8 * 8 + e;
            const float2 c2 = cs[e];
            const float x0 = x[e] * rn * gain[d], x1 = x[8 + e] * rn * gain[d + 64];
            x[e] = x0 * c2.x - x1 * c2.y;
            x[8 + e] = x1 * c2.x + x0 * c2.y;
          }
        }
      }
      *reinterpret_cast<uint4*>(dst + sw_chunk(drow, c8)) = pack8(x);
      *reinterpret_cast<uint4*>(dst + hstride + sw_chunk(drow, c8)) = pack8(x + 8);
    }
    named_bar_sync(1, kPdCompute);   // the landing area is reused by the next set
  }
}

// the 50-token chunk of one observation gets staging code with the token count folded in
#define PD_STAGE(fn, ...)          \
  do {                             \
    if (a.T == 50)                 \
      fn<50>(__VA_ARGS__);         \
    else                           \
      fn<0>(__VA_ARGS__);          \
  } while (0)

__global__ void __launch_bounds__(kPdThreads, 1)
    denoise_persistent_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmO,
                              const __grid_constant__ CUtensorMap tmGU, const __grid_constant__ CUtensorMap tmD,
                              const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                              const __grid_constant__ PdArgs a) {
  using SM = PdSmem;
  constexpr int NST = kPdStages;
  extern __shared__ uint8_t pd_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pd_smem_raw) + 1023) & ~uintptr_t(1023));
  if (smem - pd_smem_raw > static_cast<ptrdiff_t>(SM::kSlack)) {   // never expected: refuse, and release the grid
    if (threadIdx.x == 0) {
      raise_error(a.err, kErrBounds);
      atomicExch(a.sync + 1, 1u);
    }
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kOffBar);
  uint64_t* ring_full = bars;              // [NST] TMA landed
  uint64_t* ring_empty = bars + NST;       // [NST] the MMAs that read the stage completed
  uint64_t* btile_full = bars + 2 * NST;   // activation tiles of this GEMM phase staged
  uint64_t* acc_full = btile_full + 1;     // [2] accumulator segment complete
  uint64_t* q_ready = acc_full + 2;        // Q (and the suffix K/V) staged
  uint64_t* s_full = q_ready + 1;          // [2]
  uint64_t* s_free = s_full + 2;           // [2]
  uint64_t* p_full = s_free + 2;           // [2] P_i in buffer i % 2 (and O corrected)
  uint64_t* pv_done = p_full + 2;          // [2] PV_i (which read buffer i % 2) finished
  uint64_t* drain = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sx = reinterpret_cast<float*>(smem + SM::kOffMisc);   // [64]
  float* sred = sx + 64;                                        // [8]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.n_q / a.n_kv;
  const int qd = a.n_q * 128, kvd = a.n_kv * 128;
  const int nA = (a.P + 63) >> 6;                 // prefix blocks; block nA is the suffix
  const int n_items = a.n_kv * a.splits;
  const bool has_item = static_cast<int>(blockIdx.x) < n_items;
  const int item = blockIdx.x;
  const int kvg = has_item ? item / a.splits : 0;
  const int jb0 = has_item ? (item - kvg * a.splits) * a.bps : 0;
  const int jb1 = has_item ? min(nA + 1, jb0 + a.bps) : 0;
  const int nb = jb1 - jb0;
  const int npre = max(0, min(jb1, nA) - jb0);    // prefix blocks of this item
  const bool has_sfx = has_item && jb1 > nA;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], 1);
    }
    mbar_init(btile_full, 1);
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_full[1], 1);
    mbar_init(q_ready, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;   // GEMM segments at columns 0 / 64; attention S_0 0, S_1 64, O 128

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQKV);
      tma_prefetch_desc(&tmO);
      tma_prefetch_desc(&tmGU);
      tma_prefetch_desc(&tmD);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol_w = policy_evict_first(), pol_kv = policy_evict_last();
      uint32_t rs = 0;
      bool ok = true;
      auto acquire = [&](uint32_t seq) -> int {
        const int st = seq % NST;
        if (seq >= static_cast<uint32_t>(NST) && !mbar_wait(&ring_empty[st], ((seq / NST) - 1) & 1, abort_flag))
          return -1;
        return st;
      };
      for (int k = 0; ok && k < a.steps; ++k)
        for (int l = 0; ok && l < a.L; ++l)
          for (int ph = 0; ok && ph < 5; ++ph) {
            if (ph == 1) {
              for (int b = 0; ok && b < npre; ++b) {
                const int row = (l * a.n_kv + kvg) * a.P + (jb0 + b) * 64;
                for (int kv = 0; kv < 2; ++kv) {
                  const int st = acquire(rs);
                  if (st < 0) {
                    ok = false;
                    break;
                  }
                  uint8_t* dst = smem + SM::kOffRing + st * SM::kStage;
                  const CUtensorMap* m = kv ? &tmV : &tmK;
                  mbar_arrive_expect_tx(&ring_full[st], SM::kStage);
                  tma_load_2d(dst, m, &ring_full[st], 0, row, pol_kv);
                  tma_load_2d(dst + 8192, m, &ring_full[st], 64, row, pol_kv);
                  ++rs;
                }
              }
              continue;
            }
            int tiles, nkb, rpl, p0, p1;
            pd_geom(a, ph, tiles, nkb, rpl);
            pd_range(tiles * nkb, blockIdx.x, gridDim.x, p0, p1);
            const CUtensorMap* m = ph == 0 ? &tmQKV : (ph == 2 ? &tmO : (ph == 3 ? &tmGU : &tmD));
            for (int p = p0; p < p1; ++p) {
              const int st = acquire(rs);
              if (st < 0) {
                ok = false;
                break;
              }
              const int tile = p / nkb, kb = p - tile * nkb;
              mbar_arrive_expect_tx(&ring_full[st], SM::kStage);
              tma_load_2d(smem + SM::kOffRing + st * SM::kStage, m, &ring_full[st], kb * 64, l * rpl + tile * 128,
                          pol_w);
              ++rs;
            }
          }
      if (!ok) {
        *abort_flag = 1;
        raise_error(a.err, kErrTimeoutProducer);
        atomicExch(a.sync + 1, 1u);
      }
      // copies in flight land before the CTA exits
      for (uint32_t q = rs >= static_cast<uint32_t>(NST) ? rs - NST : 0; q < rs; ++q)
        if (!mbar_wait(&ring_full[q % NST], (q / NST) & 1, nullptr, kDrainTimeoutNs)) raise_error(a.err, kErrDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_g = idesc_bf16_f32(128, 64);
      const uint32_t idesc_s = idesc_bf16_f32(128, 64);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 128) | (1u << 16);   // B (V) is MN-major
      uint32_t rs = 0, n_gemm = 0, n_att = 0, blk = 0;
      bool ok = true;
      auto mmark = [&](int k, int l, int ph, int slot) {
        if (a.trace) {
          const size_t q = 1 + static_cast<size_t>(k) * (5 * a.L + 1) + l * 5 + ph;
          a.trace[(q * gridDim.x + blockIdx.x) * kPdTraceSlots + slot] = globaltimer();
        }
      };
      auto full_stage = [&](uint32_t seq) -> int {
        const int st = seq % NST;
        if (!mbar_wait(&ring_full[st], (seq / NST) & 1, abort_flag)) return -1;
        return st;
      };
      const uint32_t qa = smem_u32(smem + SM::kOffQ), pa = smem_u32(smem + SM::kOffP);
      for (int k = 0; ok && k < a.steps; ++k)
        for (int l = 0; ok && l < a.L; ++l)
          for (int ph = 0; ok && ph < 5; ++ph) {
            if (ph == 1) {
              if (!has_item) continue;
              if (!mbar_wait(q_ready, n_att & 1, abort_flag)) {
                ok = false;
                break;
              }
              ++n_att;
              mmark(k, l, ph, 6);
              tc_fence_after();
              const uint32_t rs0 = rs;
              auto pv = [&](int b) -> bool {
                const uint32_t i = blk + b;
                if (!mbar_wait(&p_full[i & 1], (i >> 1) & 1, abort_flag)) return false;
                uint32_t vaddr;
                int vst = -1;
                if (b < npre) {
                  vst = full_stage(rs0 + 2 * b + 1);
                  if (vst < 0) return false;
                  vaddr = smem_u32(smem + SM::kOffRing + vst * SM::kStage);
                } else {
                  vaddr = smem_u32(smem + SM::kOffSV);
                }
                tc_fence_after();
                const uint32_t pb = pa + (i & 1) * 16384;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                  umma_bf16(tmem + 128, sw128_kmajor_desc(pb + ks * 32), sw128_mnmajor_desc(vaddr + ks * 2048, 8192),
                            idesc_pv, (b > 0 || ks > 0) ? 1u : 0u);
                umma_commit(&pv_done[i & 1]);
                if (vst >= 0) umma_commit(&ring_empty[vst]);
                if (b == 0) mmark(k, l, 1, 15);
                return true;
              };
              for (int b = 0; ok && b < nb; ++b) {
                const uint32_t i = blk + b;
                const int sb = i & 1;
                uint32_t kaddr;
                int kst = -1;
                if (b < npre) {
                  kst = full_stage(rs0 + 2 * b);
                  if (kst < 0) {
                    ok = false;
                    break;
                  }
                  kaddr = smem_u32(smem + SM::kOffRing + kst * SM::kStage);
                } else {
                  kaddr = smem_u32(smem + SM::kOffSK);
                }
                if (i >= 2 && !mbar_wait(&s_free[sb], ((i >> 1) - 1) & 1, abort_flag)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                  umma_bf16(tmem + sb * 64, sw128_kmajor_desc(qa + (ks >> 2) * 16384 + (ks & 3) * 32),
                            sw128_kmajor_desc(kaddr + (ks >> 2) * 8192 + (ks & 3) * 32), idesc_s, ks > 0 ? 1u : 0u);
                umma_commit(&s_full[sb]);
                if (kst >= 0) umma_commit(&ring_empty[kst]);
                if (b >= 1 && !pv(b - 1)) {
                  ok = false;
                  break;
                }
              }
              if (ok && nb > 0) ok = pv(nb - 1);
              mmark(k, l, ph, 7);
              blk += nb;
              rs += 2 * npre;
              continue;
            }
            int tiles, nkb, rpl, p0, p1;
            pd_geom(a, ph, tiles, nkb, rpl);
            pd_range(tiles * nkb, blockIdx.x, gridDim.x, p0, p1);
            if (p0 >= p1) continue;
            if (!mbar_wait(btile_full, n_gemm & 1, abort_flag)) {
              ok = false;
              break;
            }
            ++n_gemm;
            mmark(k, l, ph, 6);
            tc_fence_after();
            int seg = 0, seg_start = p0, cur_tile = p0 / nkb;
            for (int p = p0; p < p1; ++p) {
              const int tile = p / nkb;
              if (tile != cur_tile) {
                umma_commit(&acc_full[seg]);
                ++seg;
                cur_tile = tile;
                seg_start = p;
              }
              const int st = full_stage(rs);
              if (st < 0) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t wa = smem_u32(smem + SM::kOffRing + st * SM::kStage);
              const uint32_t ba = smem_u32(smem + SM::kOffWork + (p - p0) * SM::kBTile);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tmem + seg * 64, sw128_kmajor_desc(wa + ks * 32), sw128_kmajor_desc(ba + ks * 32), idesc_g,
                          (p > seg_start || ks > 0) ? 1u : 0u);
              umma_commit(&ring_empty[st]);
              ++rs;
            }
            if (ok) umma_commit(&acc_full[seg]);
            mmark(k, l, ph, 7);
          }
      if (!ok) {
        *abort_flag = 1;
        raise_error(a.err, kErrTimeoutMma);
        atomicExch(a.sync + 1, 1u);
      }
      // every issued MMA completes before TMEM is released
      umma_commit(drain);
      if (!mbar_wait(drain, 0, nullptr, kWaitTimeoutNs + kDrainTimeoutNs)) raise_error(a.err, kErrDrain);
    }
  } else {
    // ------------------------------------------------------------ staging / softmax / reduction warps
    const int ct = threadIdx.x - 64;                 // 0..255
    const int lane_base = (warp & 3) * 32;           // TMEM lane quarter of this warp
    const int half = (warp - 2) >> 2;                // 0: warps 2-5, 1: warps 6-9 (when present)
    const int r = lane_base + lane;                  // TMEM lane owned by this thread
    const uint32_t tl = tmem + (static_cast<uint32_t>(lane_base) << 16);
    const float inv_Ha = 1.0f / a.Ha;
    float* ssq_attn = a.ssq;
    float* ssq_mlp = a.ssq + a.T;
    uint32_t gen = 0, acc_use[2] = {0u, 0u}, blk = 0;
    bool ok = true;
    auto csync = [] { named_bar_sync(1, kPdCompute); };
    // one lane waits, the whole warp gets the same answer (the warp-collective TMEM loads that follow
    // are then taken by all of its lanes or by none); a failed wait raises the CTA abort flag
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      int good = 1;
      if (lane == 0) good = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) *abort_flag = 1;
      return good != 0;
    };
    auto mark = [&](int slot) {
      if (a.trace && ct == 0) a.trace[(static_cast<size_t>(gen) * gridDim.x + blockIdx.x) * kPdTraceSlots + slot] = globaltimer();
    };
    auto mk_row = [&]() -> unsigned long long* {
      return a.trace ? a.trace + (static_cast<size_t>(gen) * gridDim.x + blockIdx.x) * kPdTraceSlots : nullptr;
    };

    // Every compute thread calls this after every phase, whatever happened in it, so the named
    // barriers always see all 256 threads; the result is the CTA abort flag, read after the last
    // named barrier (the same value in every thread).
    auto grid_sync = [&]() -> bool {
      named_bar_sync(1, kPdCompute);
      ++gen;
      if (ct == 0 && *abort_flag == 0) {
        __threadfence();
        if (a.trace) a.trace[(static_cast<size_t>(gen - 1) * gridDim.x + blockIdx.x) * kPdTraceSlots + 4] = globaltimer();
        atomicAdd(a.sync, 1u);
        if (a.trace) a.trace[(static_cast<size_t>(gen - 1) * gridDim.x + blockIdx.x) * kPdTraceSlots + 5] = globaltimer();
        const unsigned target = gen * gridDim.x;
        const uint64_t t0 = globaltimer();
        for (uint32_t it = 0;; ++it) {
          if (ld_acquire_u32(a.sync) >= target) break;
          if ((it & 15u) == 15u) {
            if (*reinterpret_cast<volatile unsigned*>(a.sync + 1) != 0u || globaltimer() - t0 > kWaitTimeoutNs) {
              *abort_flag = 1;
              break;
            }
          }
        }
        __threadfence();
      }
      if (ct == 0 && *abort_flag) atomicExch(a.sync + 1, 1u);   // release the other CTAs at once
      named_bar_sync(1, kPdCompute);
      return *abort_flag == 0;
    };
    // zero [0, n) floats of `p`, this CTA's share, 16-byte stores
    auto zero_share = [&](float* p, int n) {
      int i0, i1;
      pd_range(n >> 2, blockIdx.x, gridDim.x, i0, i1);
      for (int i = i0 + ct; i < i1; i += kPdCompute) reinterpret_cast<float4*>(p)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    };

    // (A, D) bf16(g * h) for pairs [p0, p0 + np); weight tile 0 also adds sum h^2 into ssq
    auto btiles_ready = [&] {
      fence_async_smem();
      tc_fence_before();
      csync();
      if (ct == 0) mbar_arrive(btile_full);
      mark(1);
    };
    // accumulator segments -> fp32 reductions into dst[t][feature]; this thread: feature row r,
    // tokens [32 half, 32 half + 32)
    auto reduce_out = [&](int p0, int p1, int nkb, float* dst, int ld) -> bool {
      int seg = 0;
      for (int tt = p0 / nkb; tt <= (p1 - 1) / nkb; ++tt, ++seg) {
        if (!warp_wait(&acc_full[seg], acc_use[seg] & 1)) return false;
        ++acc_use[seg];
        if (seg == 0) mark(2);
        tc_fence_after();
        float* col = dst + tt * 128 + r;
#pragma unroll 1
        for (int hc = half; hc < 2; hc += kPdHalves) {
          float v[32];
          tmem_ld32(tl + seg * 64 + hc * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = hc * 32 + j;
            if (t < a.T) atomicAdd(col + static_cast<size_t>(t) * ld, v[j]);
          }
        }
      }
      tc_fence_before();
      return true;
    };
    auto step_phase = [&](int k_out, int k_in) {
      if (static_cast<int>(blockIdx.x) < a.T) {
        StepArgs s = a.step;
        s.k_out = k_out;
        s.k_in = k_in;
        step_token(s, blockIdx.x, ct, kPdCompute, sx, sred, reinterpret_cast<float*>(smem + SM::kOffLandG), csync);
      }
    };
    // ---- attention of one (KV head, key split) item
    auto attention = [&](int l) -> bool {
      const PdLayer& ly = a.layers[l];
      const int GT = G * a.T;
      PD_STAGE(pd_stage_qkv, a, smem, ct, l, kvg, has_sfx, mk_row());
      fence_async_smem();
      tc_fence_before();
      csync();
      if (ct == 0) mbar_arrive(q_ready);
      mark(1);

      float m_ref = -__int_as_float(0x7f800000), l_run = 0.f;
      if (half == 0) {   // softmax: warps 2-5, one thread per query row
        for (int b = 0; b < nb; ++b) {
          const uint32_t i = blk + b;
          const int sb = i & 1;
          if (!warp_wait(&s_full[sb], (i >> 1) & 1)) break;
          if (b == 0) mark(2);
          if (b < 2) mark(10 + 2 * b);
          tc_fence_after();
          const int jj = jb0 + b;
          const int nvalid = jj < nA ? min(64, a.P - jj * 64) : a.T;
          float mx = -__int_as_float(0x7f800000);
#pragma unroll 1
          for (int hc = 0; hc < 2; ++hc) {   // pass 1: the block max over the valid keys
            float sv[32];
            tmem_ld32(tl + sb * 64 + hc * 32, sv);
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (hc * 32 + q < nvalid) mx = fmaxf(mx, sv[q]);
          }
          const float m_blk = mx * a.scale_log2;
          const bool move = m_blk > m_ref + 8.f;   // also true on the first block
          const float m_new = move ? m_blk : m_ref;
          const float alpha = move ? exp2f(m_ref - m_new) : 1.f;
          const bool any_move = __any_sync(0xffffffffu, move);
          // P buffer i % 2 is free once PV_{i-2} completed
          if (i >= 2 && !warp_wait(&pv_done[sb], ((i >> 1) - 1) & 1)) break;
          uint8_t* ps = smem + SM::kOffP + sb * 16384;
          float sum = 0.f;
#pragma unroll 1
          for (int hc = 0; hc < 2; ++hc) {   // pass 2: P = 2^(s scale - m) in bf16, the row sum
            float sv[32];
            tmem_ld32(tl + sb * 64 + hc * 32, sv);
            uint32_t pk[16];
#pragma unroll
            for (int q = 0; q < 32; q += 2) {
              const int kq = hc * 32 + q;
              const float e0 = kq < nvalid ? ex2_fast(fmaf(sv[q], a.scale_log2, -m_new)) : 0.f;
              const float e1 = kq + 1 < nvalid ? ex2_fast(fmaf(sv[q + 1], a.scale_log2, -m_new)) : 0.f;
              sum += e0 + e1;
              pk[q >> 1] = bf2(e0, e1);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4*>(ps + sw_chunk(r, hc * 4 + c)) =
                  make_uint4(pk[c * 4], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
          }
          // S buffer consumed: the MMA warp may overwrite it with S_{i+2}
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[sb]);
          l_run = l_run * alpha + sum;
          m_ref = m_new;
          // O is rescaled only after PV_{i-1}
          if (b >= 1 && any_move) {
            if (!warp_wait(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1)) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              float o[32];
              tmem_ld32(tl + 128 + c * 32, o);
#pragma unroll
              for (int q = 0; q < 32; ++q) o[q] *= alpha;
              tmem_st32(tl + 128 + c * 32, o);
            }
            tmem_wait_st();
          }
          fence_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[sb]);
          if (b < 2) mark(11 + 2 * b);
        }
      }
      if (nb > 0) {
        // all eight warps read O: (row r, 64 of the 128 columns); (m, l) of the row via shared memory
        // (m, l) of each row pass to the other half through the Q tile: the last S MMA, the last
        // reader of Q, completed before the softmax finished
        float2* sml = reinterpret_cast<float2*>(smem + SM::kOffQ);
        const uint32_t il = blk + nb - 1;
        if (half == 0) sml[r] = make_float2(m_ref, l_run);
        csync();
        if (ct == 0 && *abort_flag == 0 && !mbar_wait(&pv_done[il & 1], (il >> 1) & 1, abort_flag)) *abort_flag = 1;
        csync();
        if (*abort_flag) return false;
        mark(14);
        tc_fence_after();
        const float2 ml = sml[r];
        const float inv = 1.f / ml.y;
        const size_t mine = static_cast<size_t>(item) * 128 + r;
#pragma unroll 1
        for (int c = half * (4 / kPdHalves); c < (half + 1) * (4 / kPdHalves); ++c) {
          float o[32];
          tmem_ld32(tl + 128 + c * 32, o);
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] *= inv;
          if (r < GT) st_bf16x32(a.part_o + mine * 128 + c * 32, o);
        }
        if (r < GT && half == 0) a.part_ml[mine] = ml;
        tc_fence_before();
      }
      blk += nb;
      return true;
    };

    // ---- the schedule
    mark(0);
    step_phase(-1, 0);
    zero_share(a.acc_qkv, a.T * a.QR);
    if (blockIdx.x == 0 && ct < 2 * a.T) a.ssq[ct] = 0.f;
    ok = grid_sync();
    for (int k = 0; ok && k < a.steps; ++k) {
      for (int l = 0; ok && l < a.L; ++l) {
        const PdLayer& ly = a.layers[l];
        for (int ph = 0; ok && ph < 5; ++ph) {
          mark(0);
          if (ph == 1) {
            if (has_item && !attention(l)) *abort_flag = 1;
            mark(3);
            ok = grid_sync();
            continue;
          }
          int tiles, nkb, rpl, p0, p1;
          pd_geom(a, ph, tiles, nkb, rpl);
          pd_range(tiles * nkb, blockIdx.x, gridDim.x, p0, p1);
          const int np = p1 - p0;
          if (np > 0) {
            if (ph == 0) PD_STAGE(pd_stage_norm, a, smem, ct, p0, np, nkb, ly.attn_norm, ssq_attn, mk_row());
            else if (ph == 2) PD_STAGE(pd_stage_attn_out, a, smem, ct, p0, np, nkb, mk_row());
            else if (ph == 3) PD_STAGE(pd_stage_norm, a, smem, ct, p0, np, nkb, ly.mlp_norm, ssq_mlp, mk_row());
            else PD_STAGE(pd_stage_swiglu, a, smem, ct, p0, np, nkb, mk_row());
            btiles_ready();
          }
          // scratch of the other half of the layer, idle in this phase
          if (ph == 0) {
            zero_share(a.acc_gu, a.T * 2 * a.Ia);
            if (blockIdx.x == 0 && ct < a.T) ssq_mlp[ct] = 0.f;
          } else if (ph == 2) {
            zero_share(a.acc_qkv, a.T * a.QR);
            if (blockIdx.x == 0 && ct < a.T) ssq_attn[ct] = 0.f;
          }
          if (np > 0) {
            float* dst = ph == 0 ? a.acc_qkv : (ph == 3 ? a.acc_gu : a.h);
            const int ld = ph == 0 ? a.QR : (ph == 3 ? 2 * a.Ia : a.Ha);
            if (!reduce_out(p0, p1, nkb, dst, ld)) *abort_flag = 1;
          }
          mark(3);
          ok = grid_sync();
        }
      }
      if (!ok) break;
      mark(0);
      step_phase(k, k + 1 < a.steps ? k + 1 : -1);
      mark(3);
      if (k + 1 < a.steps) ok = grid_sync();
    }
    if (!ok) {
      *abort_flag = 1;
      raise_error(a.err, kErrTimeoutEpilogue);
      atomicExch(a.sync + 1, 1u);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace dm0
