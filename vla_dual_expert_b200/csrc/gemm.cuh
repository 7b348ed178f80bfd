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
  kModeResid = 2,     // h += acc; xn = bf16(gain_next * h); ssq_out += sum(h^2)
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
  // input row scale: inv_rms(token) = rsqrt(ssq_in[token] * inv_hidden + eps); null -> 1
  const float* ssq_in;
  float inv_hidden, eps;
  // split-K accumulation target (swap, QKV / SwiGLU / StoreF32): acc[token * ld_acc + feature]
  float* acc;
  int ld_acc;
  int* counters;      // one per 128-feature tile, zero between launches
  // kModeResid
  float* h;           // [tokens][H] fp32 residual stream
  int H;
  __nv_bfloat16* xn;  // [tokens][H] bf16(gain_next * h) for the next norm (null: skip)
  const float* gain_next;
  float* ssq_out;     // [tokens] sum of squares of h (null: skip)
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
  // kModeSwiGLU
  __nv_bfloat16* act; // [tokens][inter]
  int inter;
  // kModeStoreF32
  float* out_f32;     // normal: [M][N]
};

constexpr int kGemmThreads = 192;
constexpr int kTileLd = 129;   // padded row stride (floats) of the smem staging tile

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr uint32_t kA = 128 * 128;   // 128 rows x 64 bf16
  static constexpr uint32_t kB = BN * 128;
  static constexpr uint32_t kStage = kA + kB;
  static constexpr uint32_t kPipe = STAGES * kStage;
  static constexpr uint32_t kTile = 128 * kTileLd * 4;
  static_assert(kPipe >= kTile, "staging tile must fit in the pipeline buffers");
  static constexpr uint32_t kBytes = kPipe + 256 + 1024;   // + barriers + alignment slack
  static constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
};

// ---------------------------------------------------------------- epilogue on one 128-column group
//
// Rows are tokens, the 128 columns are output features [col0, col0 + 128).
// Warp `wid` (0..3) handles rows wid, wid + 4, ...; lane L holds columns
// L + 32 i, i = 0..3.  `src` is either the smem staging tile (normal) or the
// global split-K target (swap, read through L2).
template <bool kGlobal>
__device__ __forceinline__ void finalize_group(const GemmArgs& a, float* src, int ld, int tok0, int nrows, int col0,
                                               int wid, int lane) {
  const int D = a.head_dim;
  for (int r = wid; r < nrows; r += 4) {
    const int tok = tok0 + r;
    float x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float* p = src + static_cast<size_t>(r) * ld + lane + 32 * i;
      x[i] = kGlobal ? __ldcg(p) : *p;
    }
    if (a.mode == kModeResid) {
      float sq = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = col0 + lane + 32 * i;
        float* hp = a.h + static_cast<size_t>(tok) * a.H + col;
        float hv = x[i];
        if (!kGlobal) {
          hv += *hp;
          *hp = hv;
        }
        sq += hv * hv;
        if (a.xn) a.xn[static_cast<size_t>(tok) * a.H + col] = __float2bfloat16_rn(a.gain_next[col] * hv);
      }
      if (a.ssq_out) {
        sq = warp_sum(sq);
        if (lane == 0) atomicAdd(a.ssq_out + tok, sq);
      }
      continue;
    }
    if (a.mode == kModeStoreF32) {
      if (!kGlobal) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          a.out_f32[static_cast<size_t>(tok) * a.N + col0 + lane + 32 * i] = x[i];
      }
      continue;
    }
    // QKV and SwiGLU consume the pending RMSNorm's 1/rms of this token
    float s = 1.f;
    if (a.ssq_in) s = rsqrtf(__ldcg(a.ssq_in + tok) * a.inv_hidden + a.eps);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] *= s;
    if (kGlobal) {   // leave the split-K target zeroed for the next launch
#pragma unroll
      for (int i = 0; i < 4; ++i) src[static_cast<size_t>(r) * ld + lane + 32 * i] = 0.f;
    }
    if (a.mode == kModeSwiGLU) {
      // group = [64 gate rows | 64 up rows] of outputs [col0/2, col0/2 + 64)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int j = col0 / 2 + lane + 32 * i;
        a.act[static_cast<size_t>(tok) * a.inter + j] = __float2bfloat16_rn(silu_f(x[i]) * x[i + 2]);
      }
      continue;
    }
    // kModeQKV: 32-column chunks never straddle a head or a q/k/v section (D >= 32)
    const int qdim = a.n_q * D, kvdim = a.n_kv * D;
    float sq[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) sq[i] = warp_sum(x[i] * x[i]);
    const int b = tok / a.seq_len, p = tok - b * a.seq_len;
    const int pos = a.pos_offset + p;
    const int half = D >> 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int col = col0 + 32 * i + lane;
      const int sec = col < qdim ? 0 : (col < qdim + kvdim ? 1 : 2);
      const int d = col % D;
      float y = x[i];
      if (sec < 2) {
        // RMSNorm over this head's D columns: chunks i' with the same head as chunk i
        float ss = 0.f;
        const int chunks = D >> 5;             // 32-col chunks per head
        const int first = (i / chunks) * chunks;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j >= first && j < first + chunks) ss += sq[j];
        const float* g = sec == 0 ? a.q_gain : a.k_gain;
        y = y * rsqrtf(ss / D + a.eps) * g[d];
      }
      x[i] = y;   // normalised, before rotation
    }
    // RoPE (rotate-half): partner of column d is d +- D/2
    float part[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (D == 128) part[i] = x[i ^ 2];
      else if (D == 64) part[i] = x[i ^ 1];
      else part[i] = __shfl_xor_sync(0xffffffffu, x[i], 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int col = col0 + 32 * i + lane;
      const int sec = col < qdim ? 0 : (col < qdim + kvdim ? 1 : 2);
      const int d = col % D;
      float y = x[i];
      if (sec < 2) {
        const float2 cs = a.rope[static_cast<size_t>(pos) * half + (d % half)];
        y = d < half ? (y * cs.x - part[i] * cs.y) : (y * cs.x + part[i] * cs.y);
      }
      const __nv_bfloat16 o = __float2bfloat16_rn(y);
      if (sec == 0) {
        a.q_out[static_cast<size_t>(tok) * qdim + col] = o;
      } else {
        const int c2 = col - qdim - (sec == 2 ? kvdim : 0);
        const int kvh = c2 / D;
        __nv_bfloat16* dst = sec == 1 ? a.k_out : a.v_out;
        dst[((static_cast<size_t>(b) * a.n_kv + kvh) * a.kv_seq + p) * D + d] = o;
      }
    }
  }
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
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
      if (!a.swap) {
        float* tile = reinterpret_cast<float*>(smem);
        const int nrows = min(128, a.M - m_tile * 128);
        for (int g = 0; g < BN / 128; ++g) {
          const int row = lane_base + lane;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float v[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(lane_base) << 16) + g * 128 + c * 32, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) tile[row * kTileLd + c * 32 + j] = v[j];
          }
          named_bar_sync(1, 128);
          finalize_group<false>(a, tile, kTileLd, m_tile * 128, nrows, n_tile * BN + g * 128, wid, lane);
          named_bar_sync(1, 128);
        }
      } else {
        // lanes = output features, columns = tokens
        const int feat = m_tile * 128 + lane_base + lane;
        float* dst = a.mode == kModeResid ? a.h : a.acc;
        const int ld = a.mode == kModeResid ? a.H : a.ld_acc;
        const int tokbase = n_tile * BN;
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(lane_base) << 16) + c * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tok = tokbase + c * 32 + j;
            if (tok < a.tokens) atomicAdd(dst + static_cast<size_t>(tok) * ld + feat, v[j]);
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
          finalize_group<true>(a, dst + m_tile * 128, ld, 0, a.tokens, m_tile * 128, wid, lane);
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
