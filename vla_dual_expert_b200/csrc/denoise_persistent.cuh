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
// grid barrier, one TMA copy of the L2-resident sums, the operand build, the
// MMAs and one TMA bulk reduce-add of the split-K partial tile.
//
// Per layer l, five phases (T = tokens <= 61, the padded MMA N is 64):
//   A  qkv_acc[t][f]  += sum_k Wqkv[f][k] * bf16(g_attn[k] h[t][k])   split-K over all CTAs
//                       (tile-0 CTAs also add sum_k h[t][k]^2 for the pending RMSNorm)
//   B  attention: one CTA per (KV head, key split).  The CTA finishes q of
//      its G query heads (1/rms, QK-RMSNorm, RoPE at position P + t), then
//      runs 64-key blocks of the prefix cache (TMA) and, for the last split,
//      the suffix block through tcgen05: S = Q K^T and O += P V in TMEM; it
//      stores its partial O / l in bf16 with its (max, sum).  One helper CTA
//      per KV head builds that head's suffix K and V (K-RMSNorm, RoPE, 1/rms)
//      and publishes them with a flag; the suffix owner's producer copies them in.
//   C  h[t][f] += sum_k Wo[f][k] * o[t][k], the B operand o combined from the
//      key splits while it is staged (residual add by the reduce-add into h)
//   D  gu_acc[t][f] += sum_k Wgu[f][k] * bf16(g_mlp[k] h[t][k])  (+ MLP sum of squares)
//   E  h[t][f] += sum_k Wd[f][k] * bf16(silu(gate / rms) * (up / rms))
// and after layer L-1 the step boundary (velocity, Euler update, next input;
// one CTA per token).  The GEMM work of a phase, (128-row weight tile, 64-wide
// k-block) pairs in tile-major order, is cut into contiguous ranges, one per
// CTA, aligned to the weight tiles (pd_pairs) when there are at least as many
// CTAs as tiles; a range covers at most two tiles, each accumulated in its own
// 64-column TMEM segment.  The thread that spins on a grid barrier issues the
// next phase's operand copies as soon as the barrier completes (pd_issue).
//
// Warp roles (320 threads): warp 0 TMA producer (weights, prefix K/V, the
// suffix K/V from the helper), warp 1 TMEM owner and tcgen05.mma issuer (it
// starts on each staged pair as soon as its operand is ready), warps 2-9
// everything else: operand staging, the split-K epilogue (two warps per TMEM
// lane quarter, one per 32-column half), the softmax (two threads per query
// row, one per 32 keys of a block) and the grid barriers.  Every wait is
// bounded; a CTA that gives up raises the device error word and a global abort
// word that every other CTA's barrier polls, so the whole grid unwinds.
#pragma once
#include "attention_tc.cuh"
#include "elementwise.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace dm0 {

constexpr int kPdCompute = 256;                 // warps 2-9
constexpr int kPdThreads = 64 + kPdCompute;
constexpr int kPdHalves = 2;                     // warps sharing a TMEM lane quarter
constexpr int kPdStages = 4;       // 16 KB ring stages
constexpr int kPdBTiles = 6;       // staged activation tiles per GEMM phase
constexpr int kPdMaxSplits = 8;    // attention key splits per KV head
// trace marks per (phase, CTA): 0 phase start, 1 operand staged, 2 first accumulator / S tile
// ready, 3 results issued, 4 after the release fence, 5 barrier arrival, 6 MMA warp saw the
// operand, 7 MMA warp issued its last MMA of the phase
// 8 operand copies issued, 9 copies landed; attention: 10 / 12 S of block 0 / 1 read, 11 / 13 P of
// block 0 / 1 written, 14 O readout, 15 MMA warp issued PV of block 0; GEMM phases, in SM cycles
// (clock64) for finer steps than %globaltimer's: 12 phase start, 13 staging entered, 15 copies issued,
// 11 copies landed, 14 first pair's operand built, 10 staging done
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


struct PdArgs {
  int L, T, P, steps;       // layers, tokens (<= 64), prefix length, Euler steps
  int Ha, Ia, n_q, n_kv;    // head_dim is 128
  int QR;                   // (n_q + 2 n_kv) * 128
  float eps, scale_log2;
  int splits, bps;          // attention: key splits per KV head, 64-key blocks per split
  // RMSNorm gains of layer l: attn_norm0 + l norm_stride (and likewise q / k / mlp); computed, not
  // loaded, so no gain address waits on a load after a grid barrier
  const float *attn_norm0, *q_norm0, *k_norm0, *mlp_norm0;
  int norm_stride;          // floats between consecutive layers' gains
  const float2* rope;       // [position][64] (cos, sin)
  float* h;                 // [T][Ha] residual stream
  float* acc_qkv;           // [T][QR]  zero at launch
  float* acc_gu;            // [T][2 Ia]
  float* ssq;               // [2][T]: attention-norm and MLP-norm sums of squares, zero at launch
  __nv_bfloat16* part_o;    // [n_kv * splits][128 rows][128]: O / l of the split
  float2* part_ml;          // [n_kv * splits][128 rows]: (max, sum) of the split
  unsigned* sync;           // [0] barrier arrivals, [1] abort, [2 + g] suffix K/V of KV head g ready; zero at launch
  __nv_bfloat16* kv_sfx;    // [n_kv][K, V][64 keys][128] bf16, each tile in the shared-memory SW128 layout
  int* err;
  unsigned long long* trace;  // optional [phase][CTA][kPdTraceSlots] %globaltimer marks; null: off
  StepArgs step;            // x, h, W_in, b_in, final_norm, W_out, b_out, Ha, A, eps, steps, tokens, vel
  // time-modulated expert (the kernel's kMod instantiation): the per-loop tables of every step's
  // [1 + scale | shift | gate] x 2 per layer + the final [1 + scale | shift] (rows of tm_R floats), and
  // the shifts through the QKV and gate/up weights ([L][steps][QR], [L][steps][2 Ia])
  const float* tm_mod;
  const float* tm_bqkv;
  const float* tm_bgu;
  int tm_R;
  // grid barrier arrival as one release reduction (red.release.gpu) and no fence after the acquire
  // spin, instead of a full fence, an atomic add, the spin and a second full fence
  int fast_bar;
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
__host__ __device__ __forceinline__ void pd_range(int total, int c, int n, int& p0, int& p1) {
  p0 = static_cast<int>(static_cast<long long>(total) * c / n);
  p1 = static_cast<int>(static_cast<long long>(total) * (c + 1) / n);
}
// The (weight tile, k-block) pairs of one GEMM phase for CTA c of n.  With at least as many CTAs as
// tiles, every tile gets floor(n / tiles) or one more CTAs, which split its k-blocks evenly: no CTA
// straddles two tiles, so each adds one output segment (a CTA with two segments finished about
// 1 us after the rest and held every CTA at the grid barrier).  Fewer CTAs than tiles: an even
// contiguous split of all pairs.
__host__ __device__ __forceinline__ void pd_pairs(int tiles, int nkb, int c, int n, int& p0, int& p1) {
  if (n < tiles) {
    pd_range(tiles * nkb, c, n, p0, p1);
    return;
  }
  const int base = n / tiles, extra = n - base * tiles;   // the first `extra` tiles get base + 1 CTAs
  int t, j, m;
  if (c < extra * (base + 1)) {
    m = base + 1;
    t = c / m;
    j = c - t * m;
  } else {
    const int c2 = c - extra * (base + 1);
    m = base;
    t = extra + c2 / m;
    j = c2 - (t - extra) * m;
  }
  p0 = t * nkb + nkb * j / m;
  p1 = t * nkb + nkb * (j + 1) / m;
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

// TMA bulk reduce-add of a shared-memory fp32 tile into global memory (async proxy), and the fences
// that order it with the generic-proxy accesses of this and other CTAs
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// this warp's part of the operand of staged pair i is complete: make it visible to the tensor core
// and arrive on the pair's barrier (one arrival per compute warp)
__device__ __forceinline__ void pd_pair_ready(uint64_t* btf, int i, int ct) {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
  if ((ct & 31) == 0) mbar_arrive(&btf[i]);
}

// Operand staging, one function per phase type, inlined (as out-of-line calls, the 10-step loop of
// one observation took 6 % longer).  Thread 0 of the compute group
// requests the phase's L2 data with a few TMA tensor / bulk copies into a shared-memory landing
// area (after a proxy fence: other CTAs wrote that data through the generic proxy) and every
// compute thread waits on the stage mbarrier; the operand is then built from shared memory.  A
// unit of the build is one 16-byte bf16 chunk (8 values) of a staged row; unit u goes to compute
// thread u % kPdCompute, so the 8 chunks of a 64-column row segment sit in 8 adjacent lanes and a
// thread keeps the chunk index c8 = ct % 8.  Each function returns the stage barrier's next parity.
__device__ __forceinline__ void tma_load_2d_plain(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_plain(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                                 int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// contiguous copy; both addresses 16-byte aligned, bytes a multiple of 16
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void pd_stage_wait(uint64_t* sbar, uint32_t par, volatile int* abort_flag) {
  if (!mbar_wait(sbar, par, abort_flag)) *abort_flag = 1;
}

// (A, D) bf16(g * h) for pairs [p0, p0 + np); weight tile 0 also adds sum h^2 into ssq
template <int kT>
__device__ __forceinline__ uint32_t pd_stage_norm(const PdArgs& a, uint8_t* smem, int ct, int p0, int np, int nkb,
                                                  float* ssq, unsigned long long* mk, uint64_t* btf, uint64_t* sbar,
                                                  uint32_t par, volatile int* abort_flag) {
  using SM = PdSmem;
  const int T = kT > 0 ? kT : a.T;   // tokens; a compile-time constant for the common shape
  const int c8 = ct & 7;
  float* land = reinterpret_cast<float*>(smem + SM::kOffLandG);   // [np][T][64]
  float* sg = reinterpret_cast<float*>(smem + SM::kOffAux);       // [np][64]
  pd_stage_wait(sbar, par, abort_flag);
  if (mk && ct == 0) mk[9] = globaltimer();
  if (mk && ct == 0) mk[11] = clock64();
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
    if (mk && ct == 0 && i == 0) mk[14] = clock64();
    pd_pair_ready(btf, i, ct);
  }
  if (mk && ct == 0) mk[10] = clock64();
  return par ^ 1u;
}

// (C) attention output o = sum_j w_j o_j, w_j = l_j 2^(m_j - max m) / sum_j l_j 2^(m_j - max m), over
// the key splits j
// map_po: partial O as [slot][128 rows][128 dims] bf16, box {64 dims, T rows, S slots}; map_ml: (max, sum)
// as [slot][128 rows] 8-byte elements, box {T rows, S slots}: one copy each per staged pair
template <int kT>
__device__ __forceinline__ uint32_t pd_stage_attn_out(const PdArgs& a, uint8_t* smem, int ct, int np,
                                                      unsigned long long* mk, uint64_t* btf, uint64_t* sbar,
                                                      uint32_t par, volatile int* abort_flag) {
  using SM = PdSmem;
  const int T = kT > 0 ? kT : a.T;   // tokens; a compile-time constant for the common shape
  const int c8 = ct & 7;
  const int S = a.splits;
  const int nrows = np * S * T;
  const int mls = (S * T + 15) & ~15;   // (max, sum) entries per pair, padded to 128 bytes
  __nv_bfloat16* lo = reinterpret_cast<__nv_bfloat16*>(smem + SM::kOffLandG);   // [np][S][T][64]
  float2* lml = reinterpret_cast<float2*>(lo + static_cast<size_t>(nrows) * 64);   // [np][mls]: [S][T] used
  float* wts = reinterpret_cast<float*>(lml + np * mls);                          // [np][S][T]
  pd_stage_wait(sbar, par, abort_flag);
  if (mk && ct == 0) mk[9] = globaltimer();
  if (mk && ct == 0) mk[11] = clock64();
  for (int q = ct; q < np * T; q += kPdCompute) {   // normalised split weights of each (pair, token)
    const int i = q / T, t = q - i * T;
    float mx = -__int_as_float(0x7f800000);
    for (int sp = 0; sp < S; ++sp) mx = fmaxf(mx, lml[i * mls + sp * T + t].x);
    float den = 0.f;
    for (int sp = 0; sp < S; ++sp) {
      const float2 ml = lml[i * mls + sp * T + t];
      const float w = ml.y * ex2_fast(ml.x - mx);
      wts[(i * S + sp) * T + t] = w;
      den += w;
    }
    const float inv = 1.f / den;
    for (int sp = 0; sp < S; ++sp) wts[(i * S + sp) * T + t] *= inv;
  }
  named_bar_sync(1, kPdCompute);
  for (int i = 0; i < np; ++i) {
    for (int u = ct; u < T * 8; u += kPdCompute) {
      const int t = u >> 3;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int sp = 0; sp < S; ++sp) {
        const float w = wts[(i * S + sp) * T + t];
        const uint4 ov = *reinterpret_cast<const uint4*>(lo + static_cast<size_t>((i * S + sp) * T + t) * 64 + c8 * 8);
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(o2[e]);
          acc[2 * e] += w * f.x;
          acc[2 * e + 1] += w * f.y;
        }
      }
      *reinterpret_cast<uint4*>(smem + SM::kOffWork + i * SM::kBTile + sw_chunk(t, c8)) = pack8(acc);
    }
    if (mk && ct == 0 && i == 0) mk[14] = clock64();
    pd_pair_ready(btf, i, ct);
  }
  if (mk && ct == 0) mk[10] = clock64();
  return par ^ 1u;
}

// (E) SwiGLU of the gate/up sums with 1/rms of the MLP norm (kMod: plus the feature bias `bias`, the
// modulated norm's shift through the gate/up weights, in the interleaved column order)
template <int kT, bool kMod = false>
__device__ __forceinline__ uint32_t pd_stage_swiglu(const PdArgs& a, uint8_t* smem, int ct, int p0, int np, int nkb,
                                                    unsigned long long* mk, uint64_t* btf, uint64_t* sbar, uint32_t par,
                                                    volatile int* abort_flag, const float* bias = nullptr) {
  using SM = PdSmem;
  const int T = kT > 0 ? kT : a.T;   // tokens; a compile-time constant for the common shape
  const int c8 = ct & 7;
  const float inv_Ha = 1.0f / a.Ha;
  float* land = reinterpret_cast<float*>(smem + SM::kOffLandG);   // [np][T][128]: gate 64 | up 64
  float* sq = reinterpret_cast<float*>(smem + SM::kOffAux);       // [2T] both sums of squares
  pd_stage_wait(sbar, par, abort_flag);
  if (mk && ct == 0) mk[9] = globaltimer();
  if (mk && ct == 0) mk[11] = clock64();
  for (int i = 0; i < np; ++i) {
    for (int u = ct; u < T * 8; u += kPdCompute) {
      const int t = u >> 3;
      const float s = rsqrtf(sq[T + t] * inv_Ha + a.eps);
      const float4* g4 = reinterpret_cast<const float4*>(land + (i * T + t) * 128 + c8 * 8);
      const float4 ga = g4[0], gb = g4[1], ua = g4[16], ub = g4[17];
      const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
      const float uu[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
      float y[8];
      if constexpr (kMod) {
        const float* bg = bias + 128 * ((p0 + i) % nkb) + c8 * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = silu_f(gg[e] * s + __ldg(bg + e)) * (uu[e] * s + __ldg(bg + 64 + e));
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = silu_f(gg[e] * s) * (uu[e] * s);
      }
      *reinterpret_cast<uint4*>(smem + SM::kOffWork + i * SM::kBTile + sw_chunk(t, c8)) = pack8(y);
    }
    if (mk && ct == 0 && i == 0) mk[14] = clock64();
    pd_pair_ready(btf, i, ct);
  }
  if (mk && ct == 0) mk[10] = clock64();
  return par ^ 1u;
}

// Rows of Q (one attention item: G heads x T tokens) or of the suffix K and V (a helper CTA), built
// from the QKV sums.  Build unit = (row, c8): dims [8 c8, 8 c8 + 8) and their RoPE partners
// [64 + 8 c8, ...) sit in one thread; a row's 8 units are adjacent lanes, so the head's sum of
// squares is a 3-step shuffle.  kv = false: Q rows into the Q tile; kv = true: K rows 0..63 and V
// rows 64..127, written in the SW128 tile layout to `kv_out` (global) instead of shared memory.
// kMod: the sums first become acc / rms + bias (`bias` = this step's and layer's shift through the QKV
// weights), and the head RMSNorm is taken over that.
template <int kT, bool kMod = false>
__device__ __forceinline__ uint32_t pd_stage_qkv(const PdArgs& a, uint8_t* smem, int ct, int kvg, bool kv,
                                                 __nv_bfloat16* kv_out, unsigned long long* mk, uint64_t* sbar,
                                                 uint32_t par, volatile int* abort_flag, const float* bias = nullptr) {
  using SM = PdSmem;
  const int T = kT > 0 ? kT : a.T;   // tokens; a compile-time constant for the common shape
  const int c8 = ct & 7;
  const int G = a.n_q / a.n_kv, GT = G * T;
  const int qd = a.n_q * 128, kvd = a.n_kv * 128;
  const float inv_Ha = 1.0f / a.Ha;
  float* land = reinterpret_cast<float*>(smem + SM::kOffLandA);   // [128 rows][128]
  // the P buffers are idle while the operands are built: sums of squares, QK-norm gains, RoPE rows
  float* sq = reinterpret_cast<float*>(smem + SM::kOffP);             // [T] (+ padding to 16 bytes)
  float* sgq = reinterpret_cast<float*>(smem + SM::kOffP + 256);      // [128]
  float* sgk = reinterpret_cast<float*>(smem + SM::kOffP + 768);      // [128]
  float2* srope = reinterpret_cast<float2*>(smem + SM::kOffP + 1280); // [T][64] (cos, sin) at P + t
  pd_stage_wait(sbar, par, abort_flag);
  if (mk && ct == 0) mk[9] = globaltimer();
#pragma unroll 1
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
    if constexpr (kMod) {   // x <- x / rms + bias before the head norm
      if (valid) {
        const float s = rsqrtf(sq[t] * inv_Ha + a.eps);
        const int col = kv ? qd + which * kvd + kvg * 128 : (kvg * G + r / T) * 128;
        const float* bb = bias + col + c8 * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          x[e] = x[e] * s + __ldg(bb + e);
          x[8 + e] = x[8 + e] * s + __ldg(bb + 64 + e);
        }
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) ss += x[e] * x[e];
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    if (kMod && valid) {
      if (!(kv && which == 1)) {   // Q / K: RMSNorm over the head of the biased values, RoPE at P + t
        const float* gain = kv ? sgk : sgq;
        const float rn = rsqrtf(ss / 128.f + a.eps);
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
    } else if (valid) {
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
    if (!kv) {
      uint8_t* dst = smem + SM::kOffQ;
      *reinterpret_cast<uint4*>(dst + sw_chunk(r, c8)) = pack8(x);
      *reinterpret_cast<uint4*>(dst + 16384 + sw_chunk(r, c8)) = pack8(x + 8);
    } else {
      uint8_t* dst = reinterpret_cast<uint8_t*>(kv_out) + which * 16384;
      *reinterpret_cast<uint4*>(dst + sw_chunk(r & 63, c8)) = pack8(x);
      *reinterpret_cast<uint4*>(dst + 8192 + sw_chunk(r & 63, c8)) = pack8(x + 8);
    }
  }
  return par ^ 1u;
}

// step boundary of token blockIdx.x (velocity, Euler update, next input), out of line; kMod: the
// final norm's 1 + scale and shift of step k_out, the first attention norm's 1 + scale of step k_in,
// no time embedding
template <bool kMod = false>
__device__ __noinline__ void pd_step(const PdArgs& a, int k_out, int k_in, int ct, float* sx, float* sred, float* hs) {
  StepArgs s = a.step;
  s.k_out = k_out;
  s.k_in = k_in;
  if constexpr (kMod) {
    const float* fin = a.tm_mod + static_cast<size_t>(k_out >= 0 ? k_out : 0) * a.tm_R + 6 * a.L * a.Ha;
    s.final_norm = fin;
    if (k_in >= 0) s.attn_norm0 = a.tm_mod + static_cast<size_t>(k_in) * a.tm_R;
    step_token<true>(s, blockIdx.x, ct, kPdCompute, sx, sred, hs, [] { named_bar_sync(1, kPdCompute); }, fin + a.Ha);
  } else {
    step_token(s, blockIdx.x, ct, kPdCompute, sx, sred, hs, [] { named_bar_sync(1, kPdCompute); });
  }
}

// the 50-token chunk of one observation gets staging code with the token count folded in; the value
// is the stage barrier's next parity
// The operand copies of phase ph of layer l, Euler step k, for this CTA: issued by compute thread 0
// inside the grid barrier that precedes the phase, as soon as its spin ends and before the other
// compute threads are released, so the copies fly while they leave the barrier.  Each staging
// function above waits for exactly these bytes.  pr: this CTA's pair range [p0, p1) per phase; role
// of the attention phase: 1 an attention item of KV head kvg, 2 the suffix K/V helper of head kvg,
// 0 nothing to stage.  Returns whether copies were issued.  The landing areas are free: every
// compute thread passed the barrier's CTA-wide named barrier, and the previous phase's MMAs and
// bulk reductions completed before it.
template <bool kMod>
__device__ __forceinline__ bool pd_issue(const PdArgs& a, uint8_t* smem, int k, int l, int ph, const int* pr, int role,
                                         int kvg, uint64_t* sbar, const CUtensorMap* map_h, const CUtensorMap* map_po,
                                         const CUtensorMap* map_ml, const CUtensorMap* map_gu,
                                         const CUtensorMap* map_qkv, unsigned long long* mk) {
  using SM = PdSmem;
  const int T = a.T;
  if (mk) mk[13] = clock64();
  if (ph == 1) {
    if (role == 0) return false;
    const bool kv = role == 2;
    const int G = a.n_q / a.n_kv;
    const int qd = a.n_q * 128, kvd = a.n_kv * 128;
    float* land = reinterpret_cast<float*>(smem + SM::kOffLandA);
    float* sq = reinterpret_cast<float*>(smem + SM::kOffP);
    float* sgq = reinterpret_cast<float*>(smem + SM::kOffP + 256);
    float* sgk = reinterpret_cast<float*>(smem + SM::kOffP + 768);
    float2* srope = reinterpret_cast<float2*>(smem + SM::kOffP + 1280);
    const uint32_t sq_bytes = (4 * T + 15) & ~15u;
    fence_proxy_async_global();
    mbar_arrive_expect_tx(sbar, (kv ? 2 : G) * T * 512 + T * 512 + 1024 + sq_bytes);
    if (!kv) {
      for (int r = 0; r < G; ++r)   // head r of the group: rows r T .. r T + T - 1
        tma_load_2d_plain(land + r * T * 128, map_qkv, sbar, (kvg * G + r) * 128, 0);
    } else {
      for (int w = 0; w < 2; ++w)   // K rows at 0.., V rows at 64..
        tma_load_2d_plain(land + w * 64 * 128, map_qkv, sbar, qd + w * kvd + kvg * 128, 0);
    }
    bulk_load(srope, a.rope + static_cast<size_t>(a.P) * 64, T * 512, sbar);
    bulk_load(sgq, a.q_norm0 + static_cast<size_t>(l) * a.norm_stride, 512, sbar);
    bulk_load(sgk, a.k_norm0 + static_cast<size_t>(l) * a.norm_stride, 512, sbar);
    bulk_load(sq, a.ssq, sq_bytes, sbar);
  } else {
    const int p0 = pr[2 * ph], np = pr[2 * ph + 1] - p0;
    if (np <= 0) return false;
    int tiles, nkb, rpl;
    pd_geom(a, ph, tiles, nkb, rpl);
    int kb = p0 % nkb;
    fence_proxy_async_global();
    if (ph == 0 || ph == 3) {   // h rows and the norm's gains (kMod: this step's 1 + scale rows)
      const float* gain;
      if constexpr (kMod) {
        gain = a.tm_mod + static_cast<size_t>(k) * a.tm_R + 6 * l * a.Ha + (ph == 0 ? 0 : 3 * a.Ha);
      } else {
        gain = (ph == 0 ? a.attn_norm0 : a.mlp_norm0) + static_cast<size_t>(l) * a.norm_stride;
      }
      float* land = reinterpret_cast<float*>(smem + SM::kOffLandG);   // [np][T][64]
      float* sg = reinterpret_cast<float*>(smem + SM::kOffAux);       // [np][64]
      mbar_arrive_expect_tx(sbar, np * (T * 256 + 256));
      for (int i = 0; i < np; ++i) {
        tma_load_2d_plain(land + i * T * 64, map_h, sbar, kb * 64, 0);
        bulk_load(sg + i * 64, gain + kb * 64, 256, sbar);
        if (++kb == nkb) kb = 0;
      }
    } else if (ph == 2) {       // the key splits' partial O and (max, sum) rows
      const int G = a.n_q / a.n_kv, S = a.splits;
      const int nrows = np * S * T;
      const int mls = (S * T + 15) & ~15;
      __nv_bfloat16* lo = reinterpret_cast<__nv_bfloat16*>(smem + SM::kOffLandG);
      float2* lml = reinterpret_cast<float2*>(lo + static_cast<size_t>(nrows) * 64);
      mbar_arrive_expect_tx(sbar, nrows * (128 + 8));
      for (int i = 0; i < np; ++i) {
        const int hq = kb >> 1, g2 = hq / G, hh = hq - g2 * G;   // slots g2 S .. g2 S + S - 1, rows hh T ..
        tma_load_3d_plain(lo + static_cast<size_t>(i) * S * T * 64, map_po, sbar, (kb & 1) * 64, hh * T, g2 * S);
        tma_load_2d_plain(lml + i * mls, map_ml, sbar, hh * T, g2 * S);
        if (++kb == nkb) kb = 0;
      }
    } else {                    // the gate / up sums and both sums of squares
      float* land = reinterpret_cast<float*>(smem + SM::kOffLandG);   // [np][T][128]
      float* sq = reinterpret_cast<float*>(smem + SM::kOffAux);
      mbar_arrive_expect_tx(sbar, np * T * 512 + 8 * T);
      for (int i = 0; i < np; ++i) {
        tma_load_2d_plain(land + i * T * 128, map_gu, sbar, 128 * kb, 0);
        if (++kb == nkb) kb = 0;
      }
      bulk_load(sq, a.ssq, 8 * T, sbar);
    }
  }
  if (mk) {
    mk[15] = clock64();
    mk[8] = globaltimer();
  }
  return true;
}

#define PD_STAGE(fn, ...) (a.T == 50 ? fn<50>(__VA_ARGS__) : fn<0>(__VA_ARGS__))
#define PD_STAGE_M(fn, ...) (a.T == 50 ? fn<50, kMod>(__VA_ARGS__) : fn<0, kMod>(__VA_ARGS__))

// kMod: the time-modulated action expert (per-step gains, feature biases, gates and final norm from the
// tables in PdArgs); false compiles the DM0 expert.
template <bool kMod = false>
__global__ void __launch_bounds__(kPdThreads, 1)
    denoise_persistent_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmO,
                              const __grid_constant__ CUtensorMap tmGU, const __grid_constant__ CUtensorMap tmD,
                              const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                              const __grid_constant__ CUtensorMap tmAccQKV, const __grid_constant__ CUtensorMap tmH,
                              const __grid_constant__ CUtensorMap tmAccGU, const __grid_constant__ CUtensorMap tmHLd,
                              const __grid_constant__ CUtensorMap tmGULd, const __grid_constant__ CUtensorMap tmQKVLd,
                              const __grid_constant__ CUtensorMap tmPO, const __grid_constant__ CUtensorMap tmML,
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
  uint64_t* btile_full = bars + 2 * NST;   // [kPdBTiles] activation tile of staged pair i ready
  uint64_t* acc_full = btile_full + kPdBTiles;   // [2] accumulator segment complete
  uint64_t* q_ready = acc_full + 2;        // Q (and the suffix K/V) staged
  uint64_t* s_full = q_ready + 1;          // [2]
  uint64_t* s_free = s_full + 2;           // [2]
  uint64_t* p_full = s_free + 2;           // [2] P_i in buffer i % 2 (and O corrected)
  uint64_t* pv_done = p_full + 2;          // [2] PV_i (which read buffer i % 2) finished
  uint64_t* drain = pv_done + 2;
  uint64_t* stage_bar = drain + 1;         // TMA copies of a phase's operand data landed
  uint64_t* kvs_ready = stage_bar + 1;     // suffix K/V tiles copied in from the helper CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(kvs_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sx = reinterpret_cast<float*>(smem + SM::kOffMisc);   // [64]
  float* sred = sx + 64;                                        // [8]
  int* pr = reinterpret_cast<int*>(smem + SM::kOffMisc + 320);  // [5 phases][p0, p1]: this CTA's GEMM pairs

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.n_q / a.n_kv;
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
  // helper CTA of KV head (blockIdx.x - n_items): builds that head's suffix K and V each layer
  const bool kv_helper = !has_item && static_cast<int>(blockIdx.x) < n_items + a.n_kv;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], 1);
    }
    for (int i = 0; i < kPdBTiles; ++i) mbar_init(&btile_full[i], kPdCompute / 32);
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_full[1], 1);
    mbar_init(q_ready, kPdCompute / 32);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kPdCompute / 32);   // every compute warp reads its half of S
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], kPdCompute / 32);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 1);
    mbar_init(stage_bar, 1);
    mbar_init(kvs_ready, 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (int ph = 0; ph < 5; ++ph) {   // once per launch: the split-K division of every GEMM phase
      int tiles, nkb, rpl;
      pd_geom(a, ph, tiles, nkb, rpl);
      if (ph == 1) pr[2] = pr[3] = 0;
      else pd_pairs(tiles, nkb, blockIdx.x, gridDim.x, pr[2 * ph], pr[2 * ph + 1]);
    }
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
              if (ok && has_sfx) {
                // the suffix K/V tiles of this layer, built by this head's helper CTA in the same phase
                const unsigned want = 2u + static_cast<unsigned>(k * (5 * a.L + 1) + 5 * l + 1);
                const uint64_t t0 = globaltimer();
                for (uint32_t it = 0;; ++it) {
                  if (ld_acquire_u32(a.sync + 2 + kvg) >= want) break;
                  if ((it & 15u) == 15u && (*abort_flag || globaltimer() - t0 > kWaitTimeoutNs)) {
                    ok = false;
                    break;
                  }
                  __nanosleep(64);
                }
                if (ok) {
                  fence_proxy_async_global();
                  mbar_arrive_expect_tx(kvs_ready, 32768);
                  const __nv_bfloat16* src = a.kv_sfx + static_cast<size_t>(kvg) * 16384;
                  bulk_load(smem + SM::kOffSK, src, 16384, kvs_ready);
                  bulk_load(smem + SM::kOffSV, src + 8192, 16384, kvs_ready);
                }
              }
              continue;
            }
            int tiles, nkb, rpl, p0, p1;
            pd_geom(a, ph, tiles, nkb, rpl);
            p0 = pr[2 * ph], p1 = pr[2 * ph + 1];
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
      uint32_t rs = 0, n_att = 0, n_sfx = 0, blk = 0, bt_par = 0;   // bt_par bit i: parity of btile_full[i]
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
                  if (!mbar_wait(kvs_ready, n_sfx & 1, abort_flag)) {
                    ok = false;
                    break;
                  }
                  ++n_sfx;
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
            p0 = pr[2 * ph], p1 = pr[2 * ph + 1];
            if (p0 >= p1) continue;
            int seg = 0, seg_start = p0, cur_tile = p0 / nkb, kbc = p0 - cur_tile * nkb;
            for (int p = p0; p < p1; ++p) {
              if (p > p0 && ++kbc == nkb) {   // next weight tile
                kbc = 0;
                umma_commit(&acc_full[seg]);
                ++seg;
                ++cur_tile;
                seg_start = p;
              }
              const int i = p - p0;
              if (!mbar_wait(&btile_full[i], (bt_par >> i) & 1u, abort_flag)) {
                ok = false;
                break;
              }
              bt_par ^= 1u << i;
              if (i == 0) mmark(k, l, ph, 6);
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
    float* ssq_attn = a.ssq;
    float* ssq_mlp = a.ssq + a.T;
    uint32_t gen = 0, acc_use[2] = {0u, 0u}, blk = 0, stage_par = 0;
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
    // role of this CTA in the attention phase for the operand copies: 1 item, 2 suffix K/V helper, 0 none
    const int att_role = has_item ? 1 : (kv_helper ? 2 : 0);
    const int att_kvg = has_item ? kvg : (kv_helper ? static_cast<int>(blockIdx.x) - n_items : 0);
    bool stage_pending = false;   // thread 0: copies issued that no staging function has waited for yet
    // (nk, nl, nph): the phase that follows the barrier, whose operand copies thread 0 issues as soon as
    // its spin ends; nph < 0: none (the step phase, or the end)
    auto grid_sync = [&](int nk, int nl, int nph) -> bool {
      named_bar_sync(1, kPdCompute);
      ++gen;
      if (ct == 0 && *abort_flag == 0) {
        // the CTA barrier above orders every thread's writes before this thread's release (cumulativity)
        if (!a.fast_bar) __threadfence();
        if (a.trace) a.trace[(static_cast<size_t>(gen - 1) * gridDim.x + blockIdx.x) * kPdTraceSlots + 4] = globaltimer();
        if (a.fast_bar)
          asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(a.sync), "r"(1u) : "memory");
        else
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
        if (!a.fast_bar) __threadfence();   // else: the acquire load orders what follows, the CTA barrier below the rest
        if (*abort_flag == 0 && nph >= 0)
          stage_pending = pd_issue<kMod>(a, smem, nk, nl, nph, pr, att_role, att_kvg, stage_bar, &tmHLd, &tmPO, &tmML,
                                         &tmGULd, &tmQKVLd, mk_row());
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
    // accumulator segments -> fp32 tile [64 tokens][128 features] per segment in shared memory, then
    // one TMA bulk reduce-add per segment into dst[t][feature]; this thread: feature row r, tokens
    // [32 half, 32 half + 32)
    // gate (kMod, residual phases only): per output feature, applied to the partial tile before the add
    auto reduce_out = [&](int p0, int p1, int nkb, const CUtensorMap* map, const float* gate) -> bool {
      const int tt0 = p0 / nkb, nseg = (p1 - 1) / nkb - tt0 + 1;
      bool good = true;
      // the reduce tiles reuse the landing area of the operand copies: every warp must be done
      // building its operands (pairs are handed to the MMA warp per warp, and the first segment
      // can complete while another warp still converts a later pair)
      csync();
      for (int seg = 0; seg < nseg && good; ++seg) {
        if (!warp_wait(&acc_full[seg], acc_use[seg] & 1)) {
          good = false;
          break;
        }
        ++acc_use[seg];
        if (seg == 0) mark(2);
        tc_fence_after();
        float* rt = reinterpret_cast<float*>(smem + SM::kOffLandG + seg * 32768);
#pragma unroll 1
        for (int hc = half; hc < 2; hc += kPdHalves) {
          float v[32];
          tmem_ld32(tl + seg * 64 + hc * 32, v);
          if constexpr (kMod) {
            if (gate) {
              const float gv = __ldg(gate + (tt0 + seg) * 128 + r);
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] *= gv;
            }
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) rt[(hc * 32 + j) * 128 + r] = v[j];
        }
      }
      tc_fence_before();
      fence_async_smem();
      csync();
      // (earlier generic writes to the destination, the zeroing and other CTAs' sums, are ordered before
      // these async-proxy adds by the proxy fence this thread issued before the phase's operand copies)
      if (ct == 0 && *abort_flag == 0 && good) {
        for (int seg = 0; seg < nseg; ++seg)
          tma_reduce_add_2d(map, smem + SM::kOffLandG + seg * 32768, (tt0 + seg) * 128, 0);
        bulk_commit();
        bulk_wait_all();
        fence_proxy_async_global();   // the sums are in place before this CTA's barrier arrival
      }
      return good;
    };
    auto step_phase = [&](int k_out, int k_in) {
      if (static_cast<int>(blockIdx.x) < a.T)
        pd_step<kMod>(a, k_out, k_in, ct, sx, sred, reinterpret_cast<float*>(smem + SM::kOffLandG));
    };
    // kMod tables of step k, layer l
    auto mod_row = [&](int k, int l) { return a.tm_mod + static_cast<size_t>(k) * a.tm_R + 6 * l * a.Ha; };
    auto qkv_bias = [&](int k, int l) {
      return kMod ? a.tm_bqkv + (static_cast<size_t>(l) * a.steps + k) * a.QR : nullptr;
    };
    // ---- attention of one (KV head, key split) item
    auto attention = [&](int l, int k) -> bool {
      const int GT = G * a.T;
      stage_par = PD_STAGE_M(pd_stage_qkv, a, smem, ct, kvg, false, nullptr, mk_row(), stage_bar, stage_par, abort_flag,
                             qkv_bias(k, l));
      stage_pending = false;
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);   // one arrival per compute warp
      mark(1);

      // softmax: two threads per query row (warp w and w + 4 share a TMEM lane quarter), each on 32 of
      // the block's 64 keys; the row max is exchanged through shared memory once per block
      float m_ref = -__int_as_float(0x7f800000), l_run = 0.f;   // l_run: this half's share of the row sum
      // [2 blocks][2 halves][128 rows], in landing rows 112.. (Q uses rows < G T <= 112; a warp may
      // start here while others still convert Q from the landing area)
      float* xm = reinterpret_cast<float*>(smem + SM::kOffLandA + 112 * 512);
      for (int b = 0; b < nb; ++b) {
        const uint32_t i = blk + b;
        const int sb = i & 1;
        bool good = *abort_flag == 0 && warp_wait(&s_full[sb], (i >> 1) & 1);
        if (b == 0) mark(2);
        if (b < 2) mark(10 + 2 * b);
        tc_fence_after();
        const int jj = jb0 + b;
        const int nvalid = jj < nA ? min(64, a.P - jj * 64) : a.T;
        float sv[32];
        float mx = -__int_as_float(0x7f800000);
        if (good) {
          tmem_ld32(tl + sb * 64 + half * 32, sv);
#pragma unroll
          for (int q = 0; q < 32; ++q)
            if (half * 32 + q < nvalid) mx = fmaxf(mx, sv[q]);
        }
        xm[((b & 1) * 2 + half) * 128 + r] = mx;
        csync();
        mx = fmaxf(mx, xm[((b & 1) * 2 + (half ^ 1)) * 128 + r]);
        const float m_blk = mx * a.scale_log2;
        const bool move = m_blk > m_ref + 8.f;   // also true on the first block
        const float m_new = move ? m_blk : m_ref;
        const float alpha = move ? exp2f(m_ref - m_new) : 1.f;
        const bool any_move = __any_sync(0xffffffffu, move);
        // P buffer i % 2 is free once PV_{i-2} completed
        if (good && i >= 2) good = warp_wait(&pv_done[sb], ((i >> 1) - 1) & 1);
        float sum = 0.f;
        if (good) {
          uint8_t* ps = smem + SM::kOffP + sb * 16384;
          uint32_t pk[16];
#pragma unroll
          for (int q = 0; q < 32; q += 2) {
            const int kq = half * 32 + q;
            const float e0 = kq < nvalid ? ex2_fast(fmaf(sv[q], a.scale_log2, -m_new)) : 0.f;
            const float e1 = kq + 1 < nvalid ? ex2_fast(fmaf(sv[q + 1], a.scale_log2, -m_new)) : 0.f;
            sum += e0 + e1;
            pk[q >> 1] = bf2(e0, e1);
          }
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(ps + sw_chunk(r, half * 4 + c)) =
                make_uint4(pk[c * 4], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
        }
        // S buffer consumed: the MMA warp may overwrite it with S_{i+2}
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        l_run = l_run * alpha + sum;
        m_ref = m_new;
        // O (this half's 64 columns) is rescaled only after PV_{i-1}
        if (good && b >= 1 && any_move) {
          good = warp_wait(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1);
          if (good) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
              float o[32];
              tmem_ld32(tl + 128 + half * 64 + c * 32, o);
#pragma unroll
              for (int q = 0; q < 32; ++q) o[q] *= alpha;
              tmem_st32(tl + 128 + half * 64 + c * 32, o);
            }
            tmem_wait_st();
          }
        }
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
        if (b < 2) mark(11 + 2 * b);
      }
      if (nb > 0) {
        // all eight warps read O: (row r, 64 of the 128 columns); (m, l) of the row via shared memory
        // (m, l) of each row pass to the other half through the Q tile: the last S MMA, the last
        // reader of Q, completed before the softmax finished
        float2* sml = reinterpret_cast<float2*>(smem + SM::kOffQ);   // [2 halves][128 rows]
        const uint32_t il = blk + nb - 1;
        sml[half * 128 + r] = make_float2(m_ref, l_run);
        csync();
        if (ct == 0 && *abort_flag == 0 && !mbar_wait(&pv_done[il & 1], (il >> 1) & 1, abort_flag)) *abort_flag = 1;
        csync();
        if (*abort_flag) return false;
        mark(14);
        tc_fence_after();
        const float2 ml = make_float2(m_ref, sml[r].y + sml[128 + r].y);
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
    ok = grid_sync(0, 0, a.steps > 0 && a.L > 0 ? 0 : -1);
    for (int k = 0; ok && k < a.steps; ++k) {
      for (int l = 0; ok && l < a.L; ++l) {
        for (int ph = 0; ok && ph < 5; ++ph) {
          mark(0);
          if (ph != 1 && a.trace && ct == 0)
            a.trace[(static_cast<size_t>(gen) * gridDim.x + blockIdx.x) * kPdTraceSlots + 12] = clock64();
          if (ph == 1) {
            if (has_item && !attention(l, k)) *abort_flag = 1;
            if (kv_helper) {
              const int g = blockIdx.x - n_items;
              stage_par = PD_STAGE_M(pd_stage_qkv, a, smem, ct, g, true, a.kv_sfx + static_cast<size_t>(g) * 16384,
                                     mk_row(), stage_bar, stage_par, abort_flag, qkv_bias(k, l));
              stage_pending = false;
              csync();
              if (ct == 0) {
                __threadfence();
                asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(a.sync + 2 + g), "r"(gen + 1u) : "memory");
              }
            }
            mark(3);
            ok = grid_sync(k, l, 2);
            continue;
          }
          int tiles, nkb, rpl, p0, p1;
          pd_geom(a, ph, tiles, nkb, rpl);
          p0 = pr[2 * ph], p1 = pr[2 * ph + 1];
          const int np = p1 - p0;
          if (np > 0) {   // the operand copies were issued inside the barrier before this phase
            if (ph == 0) stage_par = PD_STAGE(pd_stage_norm, a, smem, ct, p0, np, nkb, ssq_attn, mk_row(), btile_full, stage_bar, stage_par, abort_flag);
            else if (ph == 2) stage_par = PD_STAGE(pd_stage_attn_out, a, smem, ct, np, mk_row(), btile_full, stage_bar, stage_par, abort_flag);
            else if (ph == 3) stage_par = PD_STAGE(pd_stage_norm, a, smem, ct, p0, np, nkb, ssq_mlp, mk_row(), btile_full, stage_bar, stage_par, abort_flag);
            else stage_par = PD_STAGE_M(pd_stage_swiglu, a, smem, ct, p0, np, nkb, mk_row(), btile_full, stage_bar, stage_par, abort_flag,
                                        kMod ? a.tm_bgu + (static_cast<size_t>(l) * a.steps + k) * 2 * a.Ia : nullptr);
            stage_pending = false;
            mark(1);
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
            const CUtensorMap* map = ph == 0 ? &tmAccQKV : (ph == 3 ? &tmAccGU : &tmH);
            const float* gate = kMod && (ph == 2 || ph == 4) ? mod_row(k, l) + (ph == 2 ? 2 : 5) * a.Ha : nullptr;
            if (!reduce_out(p0, p1, nkb, map, gate)) *abort_flag = 1;
          }
          mark(3);
          // next: the following phase of this layer, the next layer's QKV, or the step phase (no copies)
          const bool last = ph == 4 && l + 1 == a.L;
          ok = grid_sync(k, ph == 4 ? l + 1 : l, last ? -1 : (ph + 1) % 5);
        }
      }
      if (!ok) break;
      mark(0);
      step_phase(k, k + 1 < a.steps ? k + 1 : -1);
      mark(3);
      if (k + 1 < a.steps) ok = grid_sync(k + 1, 0, 0);
    }
    if (!ok) {
      *abort_flag = 1;
      raise_error(a.err, kErrTimeoutEpilogue);
      atomicExch(a.sync + 1, 1u);
    }
    // operand copies issued for a phase that an abort skipped land before the CTA exits
    if (ct == 0 && stage_pending && !mbar_wait(stage_bar, stage_par, nullptr, kDrainTimeoutNs))
      raise_error(a.err, kErrDrain);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace dm0
