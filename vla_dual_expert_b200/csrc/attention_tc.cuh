// Flash attention on tcgen05 for both attention shapes of the dual-expert layer
// (DM0 architecture notes, section 1): prefix rows over the prefix keys, and
// suffix rows over [prefix cache; suffix keys] (DM0.5 page, sections 5.1, 6.2).
// Keys come from up to two segments (A, B), each a [B][n_kv][len][128] array;
// every query row of a launch sees all keys of both.
//
// One CTA owns 128 query rows of one (sample, KV head) group; the G query heads
// sharing the KV head are packed along the rows as in attn_kernel, so every K/V
// tile serves all of them.  Per 128-key block j:
//   S_j = Q K_j^T        tcgen05.mma (M 128, N 64 keys, K 128), fp32 in TMEM,
//                        double-buffered so S_{j+1} overlaps the softmax of S_j
//   P_j = 2^(s - m)      softmax warps, one thread per row, read S from TMEM and
//                        write P (bf16) to shared memory as a K-major operand
//   O  += P_j V_j        tcgen05.mma (M 128, N 128 dims, K 64 keys); V is read
//                        in its stored [key][dim] order as an MN-major operand
// The running max is only moved (and O, l rescaled in TMEM) when a row's max
// grows by more than 2^8: p stays <= 256 in between and the final O / l uses a
// consistent reference, so the result is exact up to rounding.
//
// Warp roles (192 threads): warp 0 TMA producer for K/V, warp 1 TMEM owner and
// MMA issuer, warps 2..5 Q staging, softmax, O correction and output.  112 KB of
// shared memory, 256 TMEM columns and <= 168 registers per thread let two CTAs
// share an SM, so one CTA's softmax overlaps the other's tensor-core work.
#pragma once
#include "attention.cuh"
#include "ptx.cuh"

namespace dm0 {

constexpr int kFaThreads = 192;
// softmax warps: 4 (one thread per query row) in the two-CTAs-per-SM variant; 8 (two threads per
// row, 32 keys each) in the one-CTA-per-SM suffix variant, whose softmax is its critical path
template <int NP>
struct FaWarps {
  static constexpr int kSoftmax = NP == 2 ? 8 : 4;
  static constexpr int kThreads = 64 + 32 * kSoftmax;
};

template <int ST, int NP>
struct FaSmemT {
  static constexpr int kKeys = 64;                          // keys per block
  static constexpr uint32_t kQ = 32768;                     // 128 rows x 128 dims: two 64-column SW128 halves
  static constexpr uint32_t kKV = 16384;                    // 64 keys x 128 dims: two 8 KB SW128 halves
  static constexpr uint32_t kHalfKV = 8192;
  static constexpr uint32_t kP = 16384;                     // 128 rows x 64 keys, one SW128 block
  static constexpr int kStages = ST;                        // K/V blocks in flight
  static constexpr int kPBufs = NP;                         // P buffers
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQ;
  static constexpr uint32_t kOffV = kOffK + kStages * kKV;
  static constexpr uint32_t kOffP = kOffV + kStages * kKV;
  static constexpr uint32_t kOffX = kOffP + NP * kP;       // two-thread rows: [2][2][128] row maxima, [2][128] sums
  static constexpr uint32_t kX = NP == 2 ? 3072 : 0;
  static constexpr uint32_t kOffBar = kOffX + kX;
  static constexpr uint32_t kSlack = 256;                   // the dynamic base is 1024-aligned (no static smem)
  static constexpr uint32_t kBytes = kOffBar + 256 + kSlack;
  // barriers (K and V rings, S double buffer, P buffers, Q, drain), the TMEM slot and the abort flag
  static_assert((4 * ST + 4 + 2 * NP + 2) * 8 + 8 <= 256, "barrier area");
};
// Prefix pass: 2 K/V stages, one P buffer (112 KB): two CTAs per SM, K/V blocks shared by many CTAs
// through L2.  Suffix attention: 4 K/V stages and two P buffers (192 KB, one CTA per SM): deeper
// prefetch for the once-read prefix cache, and the softmax of block j+1 never waits for PV_j.
using FaSmem = FaSmemT<2, 1>;
constexpr int kFaDeepStages = 4;

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// MN-major operand, SWIZZLE_128B: 64 contiguous elements per 128-byte row, the
// next 64 along MN `mn_stride` bytes further, 8-row groups along K 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t mn_stride) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((mn_stride >> 4) & 0x3FFFu) << 16;   // leading byte offset: next 64 along MN
  d |= static_cast<uint64_t>(1024u >> 4) << 32;                   // stride byte offset: next 8 rows along K
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// byte offset of element (row, col) of a 128-row bf16 tile stored as 64-column SW128 halves
__device__ __forceinline__ uint32_t sw128_off(int row, int col) {
  const int half = col >> 6, c16 = (col & 63) >> 3;
  return half * 16384 + row * 128 + ((c16 ^ (row & 7)) << 4) + ((col & 7) << 1);
}

template <int ST, int NP>
__global__ void __launch_bounds__(FaWarps<NP>::kThreads, NP == 1 ? 2 : 1)
    fa_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb, const AttnArgs a) {
  constexpr int D = 128;
  using FS = FaSmemT<ST, NP>;
  extern __shared__ uint8_t fa_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fa_smem_raw) + 1023) & ~uintptr_t(1023));
  if (smem - fa_smem_raw > static_cast<ptrdiff_t>(FS::kSlack)) {   // never expected: refuse rather than overrun
    if (threadIdx.x == 0) raise_error(a.err, kErrBounds);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + FS::kOffBar);
  // K and V have their own rings: K_j's slot is free once S_j completed, V_j's only after PV_j, so
  // the next K blocks are requested a whole PV earlier than a shared K/V slot would allow
  uint64_t* k_full = bars;              // [ST] TMA landed K_j
  uint64_t* v_full = bars + ST;         // [ST] TMA landed V_j
  uint64_t* k_empty = bars + 2 * ST;    // [ST] S_j done: K slot free
  uint64_t* v_empty = bars + 3 * ST;    // [ST] PV_j done: V slot free
  uint64_t* s_full = bars + 4 * ST;     // [2] S_j in TMEM
  uint64_t* s_free = s_full + 2;        // [2] softmax finished reading S_j
  uint64_t* p_full = s_free + 2;        // [NP] P_j in buffer j % NP and O corrected
  uint64_t* pv_done = p_full + NP;      // [NP] PV_j (which read buffer j % NP) finished
  uint64_t* q_ready = pv_done + NP;
  uint64_t* drain = q_ready + 1;        // every issued MMA complete (before TMEM is released)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, grp = blockIdx.y;
  const size_t cta_lin = (static_cast<size_t>(blockIdx.z) * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  auto amark = [&](int j, int k) {
    if (a.trace && j < kAttnTraceBlocks) a.trace[(cta_lin * kAttnTraceBlocks + j) * 4 + k] = globaltimer();
  };
  const int b = grp / a.n_kv, kvh = grp - b * a.n_kv;
  const int G = a.n_q / a.n_kv;
  const int rows_total = G * a.seq_q;
  // 64-key blocks: segment A first, then segment B (a block never mixes segments); split z of
  // gridDim.z takes blocks [jb0, jb1)
  const int nA = (a.len_a + 63) >> 6, nB = (a.len_b + 63) >> 6;
  const int jb0 = blockIdx.z * a.blocks_per_split;
  const int jb1 = min(nA + nB, jb0 + a.blocks_per_split);
  const int nblk = jb1 - jb0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], FaWarps<NP>::kSoftmax);
    }
    for (int i = 0; i < NP; ++i) {
      mbar_init(&p_full[i], FaWarps<NP>::kSoftmax);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(q_ready, 4);
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
  const uint32_t tmem = *tmem_slot;   // S_0 at column 0, S_1 at 64, O at 128
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------ K/V producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if (nB) {
        tma_prefetch_desc(&tmKb);
        tma_prefetch_desc(&tmVb);
      }
      const uint64_t pol = policy_evict_last();
      // block j of K (v = 0) or V (v = 1) into slot j % ST
      auto issue = [&](int j, int v) {
        const int s = j % ST;
        const int jj = jb0 + j;   // global block index
        const bool segA = jj < nA;
        const CUtensorMap* m = v ? (segA ? &tmV : &tmVb) : (segA ? &tmK : &tmKb);
        const int row = segA ? grp * a.len_a + jj * 64 : grp * a.len_b + (jj - nA) * 64;
        uint64_t* bar = v ? &v_full[s] : &k_full[s];
        uint8_t* dst = smem + (v ? FS::kOffV : FS::kOffK) + s * FS::kKV;
        mbar_arrive_expect_tx(bar, FS::kKV);
        tma_load_2d(dst, m, bar, 0, row, pol);
        tma_load_2d(dst + FS::kHalfKV, m, bar, 64, row, pol);
      };
      // segment A written before the previous kernel (the prefix cache during the Euler loop) may be
      // requested before the dependency wait
      int nk = 0, nv = 0;   // K and V blocks issued
      if (a.a_stable)
        for (; nk < ST && nk < nblk && jb0 + nk < nA; ++nk) {
          issue(nk, 0);
          issue(nk, 1);
        }
      nv = nk;
      pdl_wait();
      for (int j = nk; j < nblk; ++j) {
        const int s = j % ST;
        const uint32_t par = ((j / ST) - 1) & 1;
        if (j >= ST && !mbar_wait(&k_empty[s], par, abort_flag)) break;
        issue(j, 0);
        nk = j + 1;
        if (j >= ST && !mbar_wait(&v_empty[s], par, abort_flag)) break;
        issue(j, 1);
        nv = j + 1;
      }
      if (nv < nblk) {
        *abort_flag = 1;
        raise_error(a.err, kErrTimeoutProducer);
      }
      // copies in flight land before the CTA exits
      for (int j = nk - ST; j < nk; ++j)
        if (j >= 0 && !mbar_wait(&k_full[j % ST], (j / ST) & 1, nullptr, kDrainTimeoutNs)) raise_error(a.err, kErrDrain);
      for (int j = nv - ST; j < nv; ++j)
        if (j >= 0 && !mbar_wait(&v_full[j % ST], (j / ST) & 1, nullptr, kDrainTimeoutNs)) raise_error(a.err, kErrDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 64);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 128) | (1u << 16);   // B (V) is MN-major
      const uint32_t qa = smem_u32(smem + FS::kOffQ);
      bool ok = mbar_wait(q_ready, 0, abort_flag);
      auto pv = [&](int i) -> bool {
        if (!mbar_wait(&p_full[i % NP], (i / NP) & 1, abort_flag)) return false;
        if (!mbar_wait(&v_full[i % ST], (i / ST) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(smem + FS::kOffP + (i % NP) * FS::kP);
        const uint32_t vb = smem_u32(smem + FS::kOffV + (i % ST) * FS::kKV);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_bf16(tmem + 128, sw128_kmajor_desc(pa + ks * 32), sw128_mnmajor_desc(vb + ks * 2048, FS::kHalfKV),
                    idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        umma_commit(&pv_done[i % NP]);
        umma_commit(&v_empty[i % ST]);
        return true;
      };
      for (int j = 0; ok && j < nblk; ++j) {
        const int s = j & 1;          // S buffer
        const int kvs = j % ST;       // K/V slot
        if (!mbar_wait(&k_full[kvs], (j / ST) & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (j >= 2 && !mbar_wait(&s_free[s], ((j >> 1) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + FS::kOffK + kvs * FS::kKV);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_bf16(tmem + s * 64, sw128_kmajor_desc(qa + (ks >> 2) * 16384 + (ks & 3) * 32),
                    sw128_kmajor_desc(kb + (ks >> 2) * FS::kHalfKV + (ks & 3) * 32), idesc_s, ks > 0 ? 1u : 0u);
        umma_commit(&s_full[s]);
        amark(j, 3);
        umma_commit(&k_empty[kvs]);
        if (j >= 1 && !pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && nblk > 0) ok = pv(nblk - 1);
      if (!ok) {
        *abort_flag = 1;
        raise_error(a.err, kErrTimeoutMma);
      }
      // every issued MMA completes before TMEM is released
      umma_commit(drain);
      if (!mbar_wait(drain, 0, nullptr, kWaitTimeoutNs + kDrainTimeoutNs)) raise_error(a.err, kErrDrain);
    }
  } else if constexpr (FaWarps<NP>::kSoftmax == 8) {
    // ------------------------------------------------ softmax / correction / output: two threads per row
    constexpr int kSM = 256;                        // softmax threads (named barrier 1)
    const int half = (warp - 2) >> 2;               // keys [32 half, 32 half + 32) of each block
    const int lane_base = (warp & 3) * 32;
    const int r = lane_base + lane;                 // TMEM lane = query row of this tile
    const uint32_t tl = tmem + (static_cast<uint32_t>(lane_base) << 16);
    const int pr = tile * 128 + r;
    const bool valid = pr < rows_total;
    const int head = valid ? kvh * G + pr / a.seq_q : 0;
    const int pos = valid ? pr % a.seq_q : 0;
    float* xm = reinterpret_cast<float*>(smem + FS::kOffX);   // [2 blocks][2 halves][128 rows]
    float* xl = xm + 512;                                     // [2 halves][128 rows]
    // one lane waits, the warp shares the answer (the TMEM loads after it are warp-collective)
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      int good = 1;
      if (lane == 0) good = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) *abort_flag = 1;
      return good != 0;
    };
    pdl_wait();
    if (half == 0) {   // Q row -> shared memory in the SW128 K-major layout
      const uint4* src = reinterpret_cast<const uint4*>(a.q + ((static_cast<size_t>(b) * a.seq_q + pos) * a.n_q + head) * D);
      uint8_t* qs = smem + FS::kOffQ;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 v = valid ? src[c] : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(qs + sw128_off(r, c * 8)) = v;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    float m_ref = -__int_as_float(0x7f800000), l_run = 0.f;   // l_run: this half's share of the row sum
    for (int j = 0; j < nblk; ++j) {
      const int s = j & 1;
      bool good = *abort_flag == 0 && warp_wait(&s_full[s], (j >> 1) & 1);
      if (threadIdx.x == 64) amark(j, 0);
      tc_fence_after();
      const int jj = jb0 + j;
      const int nvalid = jj < nA ? min(64, a.len_a - jj * 64) : min(64, a.len_b - (jj - nA) * 64);
      float sv[32];
      float mx = -__int_as_float(0x7f800000);
      if (good) {
        tmem_ld32(tl + s * 64 + half * 32, sv);
        if (nvalid < 64) {   // keys past a ragged end score -inf: weight 0, no per-key predicate below
#pragma unroll
          for (int q = 0; q < 32; ++q)
            if (half * 32 + q >= nvalid) sv[q] = -__int_as_float(0x7f800000);
        }
        float mx4[4] = {mx, mx, mx, mx};
#pragma unroll
        for (int q = 0; q < 32; q += 2) mx4[(q >> 1) & 3] = max3f(mx4[(q >> 1) & 3], sv[q], sv[q + 1]);
        mx = max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
      }
      xm[((j & 1) * 2 + half) * 128 + r] = mx;
      named_bar_sync(1, kSM);
      if (threadIdx.x == 64) amark(j, 1);
      mx = fmaxf(mx, xm[((j & 1) * 2 + (half ^ 1)) * 128 + r]);
      const float m_blk = mx * a.scale_log2;
      const bool move = m_blk > m_ref + 8.f;        // also true on the first block
      const float m_new = move ? m_blk : m_ref;
      const float alpha = move ? exp2f(m_ref - m_new) : 1.f;   // 0 on the first block
      const bool any_move = __any_sync(0xffffffffu, move);
      // P buffer j % NP is free once PV_{j-NP} completed
      if (good && j >= NP) good = warp_wait(&pv_done[j % NP], ((j / NP) - 1) & 1);
      float sum = 0.f;
      if (good) {
        uint32_t pk[16];
        float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(-m_new, -m_new);
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          const float2 x = ffma2(make_float2(sv[q], sv[q + 1]), sc2, nm2);
          const float p0 = ex2_fast(x.x);
          const float p1 = ex2_fast(x.y);
          sum2[(q >> 1) & 1] = fadd2(sum2[(q >> 1) & 1], make_float2(p0, p1));
          pk[q >> 1] = pack_bf16(p0, p1);
        }
        sum = (sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y);
        uint8_t* ps = smem + FS::kOffP + (j % NP) * FS::kP;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(ps + sw128_off(r, (half * 4 + c) * 8)) =
              make_uint4(pk[c * 4], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
      }
      // S buffer consumed: the MMA warp may overwrite it with S_{j+2}
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[s]);
      l_run = l_run * alpha + sum;
      m_ref = m_new;
      // O (this half's 64 columns) may only be rescaled after PV_{j-1}
      if (good && j >= 1 && any_move) {
        const int i = j - 1;
        good = warp_wait(&pv_done[i % NP], (i / NP) & 1);
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
      if (lane == 0) mbar_arrive(&p_full[j % NP]);
      if (threadIdx.x == 64) amark(j, 2);
    }
    if (nblk > 0) {
      xl[half * 128 + r] = l_run;
      named_bar_sync(1, kSM);
      const float l_tot = xl[r] + xl[128 + r];
      const bool good = *abort_flag == 0 && warp_wait(&pv_done[(nblk - 1) % NP], ((nblk - 1) / NP) & 1);
      if (good) {
        tc_fence_after();
        if (gridDim.z == 1) {
          const float inv = 1.f / l_tot;
          __nv_bfloat16* dst = a.o + ((static_cast<size_t>(b) * a.seq_q + pos) * a.n_q + head) * D;
          if (a.lse && half == 0 && valid) a.lse[(static_cast<size_t>(b) * a.seq_q + pos) * a.n_q + head] = m_ref + log2f(l_tot);
#pragma unroll 1
          for (int c = half * 2; c < half * 2 + 2; ++c) {
            float o[32];
            tmem_ld32(tl + 128 + c * 32, o);
            if (valid) {
              uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                d4[i] = make_uint4(pack_bf16(o[8 * i] * inv, o[8 * i + 1] * inv),
                                   pack_bf16(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                   pack_bf16(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                   pack_bf16(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
            }
          }
        } else {
          // split keys: this split's unnormalised O and (m, l) against its reference max
          const size_t mine = ((static_cast<size_t>(grp) * gridDim.x + tile) * gridDim.z + blockIdx.z) * 128 + r;
          float* po = a.part_o + mine * D;
#pragma unroll 1
          for (int c = half * 2; c < half * 2 + 2; ++c) {
            float o[32];
            tmem_ld32(tl + 128 + c * 32, o);
            float4* p4 = reinterpret_cast<float4*>(po + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) p4[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          }
          if (half == 0) a.part_ml[mine] = make_float2(m_ref, l_tot);
          __threadfence();
        }
      } else {
        *abort_flag = 1;
        raise_error(a.err, kErrTimeoutEpilogue);
      }
    }
  } else {
    // ------------------------------------------------ softmax / correction / output warps
    const int lane_base = (warp & 3) * 32;
    const int r = lane_base + lane;                 // TMEM lane = query row of this tile
    const uint32_t tl = tmem + (static_cast<uint32_t>(lane_base) << 16);
    const int pr = tile * 128 + r;
    const bool valid = pr < rows_total;
    const int head = valid ? kvh * G + pr / a.seq_q : 0;
    const int pos = valid ? pr % a.seq_q : 0;
    pdl_wait();
    {   // Q row -> shared memory in the SW128 K-major layout
      const uint4* src = reinterpret_cast<const uint4*>(a.q + ((static_cast<size_t>(b) * a.seq_q + pos) * a.n_q + head) * D);
      uint8_t* qs = smem + FS::kOffQ;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 v = valid ? src[c] : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(qs + sw128_off(r, c * 8)) = v;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    float m_ref = -__int_as_float(0x7f800000), l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const int s = j & 1;
      if (!mbar_wait(&s_full[s], (j >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int jj = jb0 + j;
      const int nvalid = jj < nA ? min(64, a.len_a - jj * 64) : min(64, a.len_b - (jj - nA) * 64);
      // the whole S row in registers: two TMEM loads, one wait
      float sv[64];
      {
        uint32_t* u = reinterpret_cast<uint32_t*>(sv);
#pragma unroll
        for (int c = 0; c < 2; ++c)
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
              "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
              "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
              : "=r"(u[c * 32 + 0]), "=r"(u[c * 32 + 1]), "=r"(u[c * 32 + 2]), "=r"(u[c * 32 + 3]),
                "=r"(u[c * 32 + 4]), "=r"(u[c * 32 + 5]), "=r"(u[c * 32 + 6]), "=r"(u[c * 32 + 7]),
                "=r"(u[c * 32 + 8]), "=r"(u[c * 32 + 9]), "=r"(u[c * 32 + 10]), "=r"(u[c * 32 + 11]),
                "=r"(u[c * 32 + 12]), "=r"(u[c * 32 + 13]), "=r"(u[c * 32 + 14]), "=r"(u[c * 32 + 15]),
                "=r"(u[c * 32 + 16]), "=r"(u[c * 32 + 17]), "=r"(u[c * 32 + 18]), "=r"(u[c * 32 + 19]),
                "=r"(u[c * 32 + 20]), "=r"(u[c * 32 + 21]), "=r"(u[c * 32 + 22]), "=r"(u[c * 32 + 23]),
                "=r"(u[c * 32 + 24]), "=r"(u[c * 32 + 25]), "=r"(u[c * 32 + 26]), "=r"(u[c * 32 + 27]),
                "=r"(u[c * 32 + 28]), "=r"(u[c * 32 + 29]), "=r"(u[c * 32 + 30]), "=r"(u[c * 32 + 31])
              : "r"(tl + s * 64 + c * 32));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      }
      // S buffer consumed: the MMA warp may overwrite it with S_{j+2}
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[s]);
      // keys past the end of a ragged last block score -inf (their weight 2^-inf is 0), so the max and
      // exponent loops below carry no per-key predicate
      const float ninf = -__int_as_float(0x7f800000);
      if (nvalid < 64) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i >= nvalid) sv[i] = ninf;
      }
      // block max, eight independent chains of three-operand maxima
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = ninf;
#pragma unroll
      for (int i = 0; i < 64; i += 2) mx8[(i >> 1) & 7] = max3f(mx8[(i >> 1) & 7], sv[i], sv[i + 1]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_blk = mx * a.scale_log2;
      const bool move = m_blk > m_ref + 8.f;        // also true on the first block
      const float m_new = move ? m_blk : m_ref;
      const float alpha = move ? exp2f(m_ref - m_new) : 1.f;   // 0 on the first block
      // P = 2^(s*scale - m), packed to bf16; the exponent arguments and the row sum (four paired
      // partial sums) in paired fp32 arithmetic
      uint32_t pk[32];
      float2 sum2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) sum2[k] = make_float2(0.f, 0.f);
      const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(-m_new, -m_new);
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        const float2 x = ffma2(make_float2(sv[i], sv[i + 1]), sc2, nm2);
        const float p0 = ex2_fast(x.x);
        const float p1 = ex2_fast(x.y);
        sum2[(i >> 1) & 3] = fadd2(sum2[(i >> 1) & 3], make_float2(p0, p1));
        pk[i >> 1] = pack_bf16(p0, p1);
      }
      const float sum = ((sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y)) +
                        ((sum2[2].x + sum2[2].y) + (sum2[3].x + sum2[3].y));
      l_run = l_run * alpha + sum;
      m_ref = m_new;
      // P buffer j % NP is free once PV_{j-NP} completed; O may only be rescaled after PV_{j-1}
      const bool any_move = __any_sync(0xffffffffu, move);
      if (j >= NP) {
        if (!mbar_wait(&pv_done[j % NP], ((j / NP) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
      }
      if (j >= 1 && (NP == 1 || any_move)) {
        const int i = j - 1;
        if (NP > 1 && !mbar_wait(&pv_done[i % NP], (i / NP) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      if (j >= 1 && any_move) {
        {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(tl + 128 + c * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tl + 128 + c * 32, o);
          }
          tmem_wait_st();
        }
      }
      uint8_t* ps = smem + FS::kOffP + (j % NP) * FS::kP;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(ps + sw128_off(r, c * 8)) =
            make_uint4(pk[c * 4], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[j % NP]);
    }
    if (!ok) {
      *abort_flag = 1;
      raise_error(a.err, kErrTimeoutEpilogue);
    } else if (nblk > 0) {
      if (mbar_wait(&pv_done[(nblk - 1) % NP], ((nblk - 1) / NP) & 1, abort_flag)) {
        tc_fence_after();
        if (gridDim.z == 1) {
          const float inv = 1.f / l_run;
          __nv_bfloat16* dst = a.o + ((static_cast<size_t>(b) * a.seq_q + pos) * a.n_q + head) * D;
          if (a.lse && valid) a.lse[(static_cast<size_t>(b) * a.seq_q + pos) * a.n_q + head] = m_ref + log2f(l_run);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(tl + 128 + c * 32, o);
            if (valid) {
              uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                d4[i] = make_uint4(pack_bf16(o[8 * i] * inv, o[8 * i + 1] * inv),
                                   pack_bf16(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                   pack_bf16(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                   pack_bf16(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
            }
          }
        } else {
          // split keys: this split's unnormalised O and (m, l) against its reference max
          const size_t mine = ((static_cast<size_t>(grp) * gridDim.x + tile) * gridDim.z + blockIdx.z) * 128 + r;
          float* po = a.part_o + mine * D;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(tl + 128 + c * 32, o);
            float4* p4 = reinterpret_cast<float4*>(po + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) p4[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          }
          a.part_ml[mine] = make_float2(m_ref, l_run);
          __threadfence();
        }
      } else {
        *abort_flag = 1;
        raise_error(a.err, kErrTimeoutEpilogue);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if (gridDim.z > 1) {
    // the last split of this (group, row tile) merges the partial states
    int* s_last = reinterpret_cast<int*>(tmem_slot + 2);
    if (threadIdx.x == 0) {
      int* ctr = a.counters + static_cast<size_t>(grp) * gridDim.x + tile;
      const int prev = atomicAdd(ctr, 1);
      *s_last = prev == static_cast<int>(gridDim.z) - 1;
      if (*s_last) *ctr = 0;
    }
    __syncthreads();
    if (*s_last && !*abort_flag) {
      __threadfence();
      const size_t slot0 = (static_cast<size_t>(grp) * gridDim.x + tile) * gridDim.z;
      combine_splits<128>(a, slot0, tile, b, kvh, reinterpret_cast<float*>(smem), threadIdx.x, FaWarps<NP>::kThreads);
    }
  }
}

}  // namespace dm0
