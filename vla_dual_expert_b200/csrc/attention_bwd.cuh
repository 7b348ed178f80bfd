// Adjoint of the merged attention of the training step on tcgen05 (DM0.5 page, section 5.3: the
// flow-matching loss is differentiated through the action expert; section 6.2: suffix rows attend to
// [prefix cache; suffix keys]).  With s = q.k / sqrt(D), p = softmax(s) and o = sum_k p v, and dO the
// gradient of the attention output:
//   dP = dO V^T,  delta = sum_d dO o,  dS = p (dP - delta) / sqrt(D),
//   dQ = dS K,    dK = dS^T Q,         dV = p^T dO.
// The probabilities are not kept from the forward: each is rebuilt as 2^(s log2(e) - lse) from the
// forward's base-2 log-sum-exp of its row.
//
// One CTA owns 128 query rows of one (sample, KV head) group: the G query heads sharing the KV head
// packed along the rows, as in the forward.  Per 64-key block j of [segment A; segment B]:
//   S_j  = Q K_j^T, dP_j = dO V_j^T   tcgen05.mma, M 128 rows, N 64 keys, K 128 dims, fp32 in TMEM
//   P_j, dS_j                         the softmax warps (one thread per row), bf16 into shared memory
//   dQ  += dS_j K_j                   M 128 rows, N 128 dims, K 64 keys; K_j read as an MN-major B
//   dV_j^T = dO^T P_j, dK_j^T = Q^T dS_j   M 128 dims, N 64 keys, K 128 rows: A = dO^T, Q^T staged once
//                                     K-major, B = P_j, dS_j read MN-major
//   the same warps then read dV_j^T and dK_j^T (TMEM lane = dimension) and add them to dK, dV in
//   global memory, 32 consecutive dimensions per warp access.
// Rows past the tile's valid rows hold zeros in Q, dO and their transposes and write P = dS = 0, so they
// add nothing to dK, dV.
//
// Warp roles (192 threads): warp 0 TMA producer of the K/V blocks, warp 1 TMEM owner and MMA issuer,
// warps 2-5 operand staging, softmax, and the dK / dV / dQ epilogues.  One CTA per SM (224 KB of
// shared memory), 384 of 512 TMEM columns.  Every wait is bounded.
#pragma once
#include "attention_tc.cuh"
#include "ptx.cuh"

namespace dm0 {

struct AttnBwdArgs {
  const __nv_bfloat16* q;    // [B][seq_q][n_q][D] (the forward's q)
  const __nv_bfloat16* o;    // [B][seq_q][n_q][D] (the forward's output)
  const float* dout;         // [B][seq_q][n_q][D] fp32: gradient of o
  const float* lse;          // [B][seq_q][n_q]: the forward's base-2 log-sum-exp per row
  int seq_q;
  int len_a, len_b;          // keys of segments A and B (their K/V come through the tensor maps)
  int n_q, n_kv;
  float scale_log2;          // log2(e) / sqrt(D)
  float scale;               // 1 / sqrt(D)
  float* dq;                 // [B][seq_q][n_q][D] fp32, written
  float* dk;                 // [B][n_kv][len_a + len_b][D] fp32, added to (zeroed by the caller)
  float* dv;
  int* err;
};

struct FaBwdSmem {
  static constexpr uint32_t kTile = 32768;                  // 128 x 128 bf16, two 64-column SW128 halves
  static constexpr uint32_t kKV = 16384;                    // 64 keys x 128 dims
  static constexpr uint32_t kHalfKV = 8192;
  static constexpr uint32_t kPS = 16384;                    // 128 rows x 64 keys, one SW128 block
  static constexpr int kStages = 2;
  static constexpr uint32_t kOffQ = 0;                      // Q: A of S (K-major, K = dims)
  static constexpr uint32_t kOffDO = kOffQ + kTile;         // dO: A of dP
  static constexpr uint32_t kOffQT = kOffDO + kTile;        // Q^T: A of dK^T (K-major, K = rows)
  static constexpr uint32_t kOffDOT = kOffQT + kTile;       // dO^T: A of dV^T
  static constexpr uint32_t kOffK = kOffDOT + kTile;
  static constexpr uint32_t kOffV = kOffK + kStages * kKV;
  static constexpr uint32_t kOffP = kOffV + kStages * kKV;
  static constexpr uint32_t kOffDS = kOffP + kPS;
  static constexpr uint32_t kOffBar = kOffDS + kPS;
  static constexpr uint32_t kSlack = 1024;                  // the dynamic base is rounded up to 1024
  static constexpr uint32_t kBytes = kOffBar + 256 + kSlack;
  static_assert(kBytes <= 232448, "shared memory per CTA");
};
constexpr int kFaBwdThreads = 192;
// TMEM columns
constexpr uint32_t kBwS = 0, kBwDP = 64, kBwDQ = 128, kBwDV = 256, kBwDK = 320, kBwCols = 512;

__global__ void __launch_bounds__(kFaBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
                  const AttnBwdArgs a) {
  constexpr int D = 128;
  constexpr int ST = FaBwdSmem::kStages;
  using FS = FaBwdSmem;
  extern __shared__ uint8_t fb_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fb_smem_raw) + 1023) & ~uintptr_t(1023));
  if (smem - fb_smem_raw > static_cast<ptrdiff_t>(FS::kSlack)) {   // never expected: refuse rather than overrun
    if (threadIdx.x == 0) raise_error(a.err, kErrBounds);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + FS::kOffBar);
  uint64_t* kv_full = bars;             // [ST] K_j and V_j landed
  uint64_t* kv_empty = bars + ST;       // [ST] every MMA reading K_j / V_j done
  uint64_t* s_full = bars + 2 * ST;     // S_j and dP_j in TMEM
  uint64_t* p_ready = s_full + 1;       // P_j, dS_j in shared memory; S / dP read
  uint64_t* g_full = p_ready + 1;       // dV_j^T, dK_j^T complete (P_j / dS_j free again)
  uint64_t* g_free = g_full + 1;        // dV_j^T, dK_j^T read by the epilogue
  uint64_t* q_ready = g_free + 1;       // Q, dO and their transposes staged
  uint64_t* drain = q_ready + 1;        // every issued MMA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, grp = blockIdx.y;
  const int b = grp / a.n_kv, kvh = grp - b * a.n_kv;
  const int G = a.n_q / a.n_kv;
  const int rows_total = G * a.seq_q;
  const int nA = (a.len_a + 63) >> 6, nB = (a.len_b + 63) >> 6;
  const int nblk = nA + nB;
  const int ntot = a.len_a + a.len_b;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_ready, 4);
    mbar_init(g_full, 1);
    mbar_init(g_free, 4);
    mbar_init(q_ready, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kBwCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
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
      pdl_wait();
      int issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % ST;
        if (j >= ST && !mbar_wait(&kv_empty[s], ((j / ST) - 1) & 1, abort_flag)) {
          *abort_flag = 1;
          raise_error(a.err, kErrTimeoutProducer);
          break;
        }
        const bool segA = j < nA;
        const CUtensorMap* mk = segA ? &tmK : &tmKb;
        const CUtensorMap* mv = segA ? &tmV : &tmVb;
        const int row = segA ? grp * a.len_a + j * 64 : grp * a.len_b + (j - nA) * 64;
        mbar_arrive_expect_tx(&kv_full[s], 2 * FS::kKV);
        uint8_t* kd = smem + FS::kOffK + s * FS::kKV;
        uint8_t* vd = smem + FS::kOffV + s * FS::kKV;
        tma_load_2d(kd, mk, &kv_full[s], 0, row, pol);
        tma_load_2d(kd + FS::kHalfKV, mk, &kv_full[s], 64, row, pol);
        tma_load_2d(vd, mv, &kv_full[s], 0, row, pol);
        tma_load_2d(vd + FS::kHalfKV, mv, &kv_full[s], 64, row, pol);
        issued = j + 1;
      }
      for (int j = issued - ST; j < issued; ++j) {   // copies in flight land before the CTA exits
        if (j < 0) continue;
        if (!mbar_wait(&kv_full[j % ST], (j / ST) & 1, nullptr, kDrainTimeoutNs)) raise_error(a.err, kErrDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 64);                 // S, dP: both operands K-major
      const uint32_t id_dq = idesc_bf16_f32(128, 128) | (1u << 16);  // dQ: B (K_j) MN-major
      const uint32_t id_g = idesc_bf16_f32(128, 64) | (1u << 16);    // dV^T, dK^T: B (P, dS) MN-major
      const uint32_t qa = smem_u32(smem + FS::kOffQ), doa = smem_u32(smem + FS::kOffDO);
      const uint32_t qta = smem_u32(smem + FS::kOffQT), dota = smem_u32(smem + FS::kOffDOT);
      const uint32_t pa = smem_u32(smem + FS::kOffP), dsa = smem_u32(smem + FS::kOffDS);
      bool ok = mbar_wait(q_ready, 0, abort_flag);
      for (int j = 0; ok && j < nblk; ++j) {
        const int s = j % ST;
        if (!mbar_wait(&kv_full[s], (j / ST) & 1, abort_flag)) {
          ok = false;
          break;
        }
        // S and dP of block j - 1 were read before this warp's wait on p_ready in iteration j - 1
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + FS::kOffK + s * FS::kKV);
        const uint32_t vb = smem_u32(smem + FS::kOffV + s * FS::kKV);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ao = (ks >> 2) * 16384 + (ks & 3) * 32, bo = (ks >> 2) * FS::kHalfKV + (ks & 3) * 32;
          umma_bf16(tmem + kBwS, sw128_kmajor_desc(qa + ao), sw128_kmajor_desc(kb + bo), id_s, ks > 0 ? 1u : 0u);
          umma_bf16(tmem + kBwDP, sw128_kmajor_desc(doa + ao), sw128_kmajor_desc(vb + bo), id_s, ks > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
        // P_j and dS_j written; the epilogue has read dV^T, dK^T of block j - 1
        if (!mbar_wait(p_ready, j & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (j >= 1 && !mbar_wait(g_free, (j - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)   // dQ += dS_j K_j over the block's 64 keys
          umma_bf16(tmem + kBwDQ, sw128_kmajor_desc(dsa + ks * 32), sw128_mnmajor_desc(kb + ks * 2048, FS::kHalfKV),
                    id_dq, (j > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {   // dV^T = dO^T P_j, dK^T = Q^T dS_j over the 128 rows
          const uint32_t ao = (ks >> 2) * 16384 + (ks & 3) * 32;
          umma_bf16(tmem + kBwDV, sw128_kmajor_desc(dota + ao), sw128_mnmajor_desc(pa + ks * 2048, FS::kPS), id_g,
                    ks > 0 ? 1u : 0u);
          umma_bf16(tmem + kBwDK, sw128_kmajor_desc(qta + ao), sw128_mnmajor_desc(dsa + ks * 2048, FS::kPS), id_g,
                    ks > 0 ? 1u : 0u);
        }
        umma_commit(g_full);
        umma_commit(&kv_empty[s]);
      }
      if (!ok) {
        *abort_flag = 1;
        raise_error(a.err, kErrTimeoutMma);
      }
      umma_commit(drain);
      if (!mbar_wait(drain, 0, nullptr, kWaitTimeoutNs + kDrainTimeoutNs)) raise_error(a.err, kErrDrain);
    }
  } else {
    // ------------------------------------------------ staging, softmax and the epilogues (warps 2..5)
    const int lane_base = (warp & 3) * 32;
    const int r = lane_base + lane;   // TMEM lane: query row (S, dP, dQ) or dimension (dV^T, dK^T)
    const uint32_t tl = tmem + (static_cast<uint32_t>(lane_base) << 16);
    const int pr = tile * 128 + r;
    const bool valid = pr < rows_total;
    const int head = valid ? kvh * G + pr / a.seq_q : 0;
    const int pos = valid ? pr % a.seq_q : 0;
    const size_t rowo = (static_cast<size_t>(b) * a.seq_q + pos) * a.n_q + head;   // row of q, o, dO, dq
    // one lane waits, the warp shares the answer (the TMEM loads after it are warp-collective)
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      int good = 1;
      if (lane == 0) good = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      return good != 0;
    };
    pdl_wait();
    // Q and dO rows K-major (A of S and dP), and the same values along K of Q^T and dO^T (A of dK^T and
    // dV^T: element (dimension d, row r)); delta = dO . o of the row in fp32
    float delta = 0.f;
    {
      uint8_t* qs = smem + FS::kOffQ;
      uint8_t* ds = smem + FS::kOffDO;
      uint8_t* qt = smem + FS::kOffQT;
      uint8_t* dt = smem + FS::kOffDOT;
      const uint4* qsrc = reinterpret_cast<const uint4*>(a.q + rowo * D);
      const uint4* osrc = reinterpret_cast<const uint4*>(a.o + rowo * D);
      const float4* dsrc = reinterpret_cast<const float4*>(a.dout + rowo * D);
#pragma unroll 1
      for (int c = 0; c < 16; ++c) {   // dimensions 8 c .. 8 c + 7
        const uint4 qv = valid ? qsrc[c] : make_uint4(0, 0, 0, 0);
        const uint4 ov = valid ? osrc[c] : make_uint4(0, 0, 0, 0);
        const float4 d0 = valid ? dsrc[2 * c] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 d1 = valid ? dsrc[2 * c + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
        const __nv_bfloat16* ob = reinterpret_cast<const __nv_bfloat16*>(&ov);
#pragma unroll
        for (int e = 0; e < 8; ++e) delta += dd[e] * __bfloat162float(ob[e]);
        const uint4 dv = make_uint4(pack_bf16(dd[0], dd[1]), pack_bf16(dd[2], dd[3]), pack_bf16(dd[4], dd[5]), pack_bf16(dd[6], dd[7]));
        *reinterpret_cast<uint4*>(qs + sw128_off(r, c * 8)) = qv;
        *reinterpret_cast<uint4*>(ds + sw128_off(r, c * 8)) = dv;
        const uint16_t* qe = reinterpret_cast<const uint16_t*>(&qv);
        const uint16_t* de = reinterpret_cast<const uint16_t*>(&dv);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          *reinterpret_cast<uint16_t*>(qt + sw128_off(c * 8 + e, r)) = qe[e];
          *reinterpret_cast<uint16_t*>(dt + sw128_off(c * 8 + e, r)) = de[e];
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    const float lse = valid ? a.lse[rowo] : 0.f;
    // dV^T and dK^T of block jb (this thread: dimension r) added to dv, dk; keys past a ragged end skipped
    auto store_grads = [&](int jb) {
      const int key0 = jb < nA ? jb * 64 : a.len_a + (jb - nA) * 64;
      const int nv = jb < nA ? min(64, a.len_a - jb * 64) : min(64, a.len_b - (jb - nA) * 64);
      float* dvp = a.dv + (static_cast<size_t>(grp) * ntot + key0) * D + r;
      float* dkp = a.dk + (static_cast<size_t>(grp) * ntot + key0) * D + r;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float gv[32], gk[32];
        tmem_ld32(tl + kBwDV + 32 * c, gv);
        tmem_ld32(tl + kBwDK + 32 * c, gk);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          if (32 * c + e < nv) {
            atomicAdd(dvp + static_cast<size_t>(32 * c + e) * D, gv[e]);
            atomicAdd(dkp + static_cast<size_t>(32 * c + e) * D, gk[e]);
          }
        }
      }
    };
    bool ok = *abort_flag == 0;
    for (int j = 0; ok && j < nblk; ++j) {
      if (!warp_wait(s_full, j & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int nvalid = j < nA ? min(64, a.len_a - j * 64) : min(64, a.len_b - (j - nA) * 64);
      // P = 2^(s log2(e)/sqrt(D) - lse), dS = P (dP - delta) / sqrt(D), both bf16; keys past a ragged
      // end and rows past the tile's valid rows give 0
      uint32_t pk[32], dk[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float sv[32], dp[32];
        tmem_ld32(tl + kBwS + 32 * hh, sv);
        tmem_ld32(tl + kBwDP + 32 * hh, dp);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int key = 32 * hh + e;
          const float p0 = (valid && key < nvalid) ? ex2_fast(fmaf(sv[e], a.scale_log2, -lse)) : 0.f;
          const float p1 = (valid && key + 1 < nvalid) ? ex2_fast(fmaf(sv[e + 1], a.scale_log2, -lse)) : 0.f;
          const float g0 = p0 * (dp[e] - delta) * a.scale, g1 = p1 * (dp[e + 1] - delta) * a.scale;
          pk[(key >> 1)] = pack_bf16(p0, p1);
          dk[(key >> 1)] = pack_bf16(g0, g1);
        }
      }
      // the MMAs of block j - 1 have read P and dS (g_full): its dV^T, dK^T go out first, then the
      // buffers take block j
      if (j >= 1) {
        if (!warp_wait(g_full, (j - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        store_grads(j - 1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(g_free);
      }
      uint8_t* ps = smem + FS::kOffP;
      uint8_t* dss = smem + FS::kOffDS;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        *reinterpret_cast<uint4*>(ps + sw128_off(r, c * 8)) = make_uint4(pk[c * 4], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
        *reinterpret_cast<uint4*>(dss + sw128_off(r, c * 8)) =
            make_uint4(dk[c * 4], dk[c * 4 + 1], dk[c * 4 + 2], dk[c * 4 + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready);
    }
    if (ok && nblk > 0) {
      if (warp_wait(g_full, (nblk - 1) & 1)) {
        tc_fence_after();
        store_grads(nblk - 1);
        // dQ of this row (the accumulation over every block is complete with the last commit)
        float* dqp = a.dq + rowo * D;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(tl + kBwDQ + 32 * c, v);
          if (valid) {
            float4* d4 = reinterpret_cast<float4*>(dqp + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      } else {
        ok = false;
      }
    }
    if (!ok) {
      *abort_flag = 1;
      raise_error(a.err, kErrTimeoutEpilogue);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwCols);
  }
}

}  // namespace dm0
