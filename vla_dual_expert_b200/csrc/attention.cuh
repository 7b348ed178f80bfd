// Merged GQA attention of the dual-expert layer (DM0 architecture notes,
// section 1; DM0.5 page, section 6.2 for the suffix reading the prefix cache).
//
// One CTA owns 128 query rows of one (sample, KV head) group: the G = n_q/n_kv
// query heads that share the KV head are packed along the row axis (row
// r -> head r / Tq, position r % Tq), so each K/V tile read from HBM serves
// every head of the group.  Keys are the concatenation of segment A (e.g. the
// cached prefix) and segment B (e.g. the fresh suffix); every row of a launch
// sees all of them, so the pages' block mask is expressed by which segments a
// launch is given (prefix rows: A = prefix; suffix rows: A = prefix cache,
// B = suffix).
//
// Online softmax (base-2 exponentials) over 64-key tiles staged with cp.async
// into XOR-swizzled shared memory; QK^T and PV on bf16 tensor cores
// (mma.m16n8k16, fp32 accumulate).  Keys may be split across CTAs
// (blockIdx.z); partial (O, m, l) go to a workspace and the last CTA of the
// group combines them.
#pragma once
#include "ptx.cuh"

namespace dm0 {

struct AttnArgs {
  const __nv_bfloat16* q;   // [B][seq_q][n_q][D]
  int seq_q;
  const __nv_bfloat16* ka;  // [B][n_kv][len_a][D]
  const __nv_bfloat16* va;
  int len_a;
  const __nv_bfloat16* kb;  // [B][n_kv][len_b][D] (len_b may be 0)
  const __nv_bfloat16* vb;
  int len_b;
  __nv_bfloat16* o;         // [B][seq_q][n_q][D]
  int n_q, n_kv;
  float scale_log2;         // log2(e) / sqrt(D)
  int blocks_per_split;     // 64-key blocks per split
  int a_stable;             // segment A predates the previous kernel: prefetch it before the PDL wait
  float* part_o;            // [slots][128][D]
  float2* part_ml;          // [slots][128]
  int* counters;            // [groups * row tiles]
  int* err;
  // tcgen05 kernel, unsplit launches only (null: off): per query row, at the row's place in o
  // ([B][seq_q][n_q]), the base-2 log-sum-exp m + log2(l) of its scaled scores (p = 2^(s * scale_log2 - lse))
  float* lse;
  // tcgen05 kernel, two-threads-per-row instance (null: off): per CTA (blockIdx linear, x fastest) and
  // 64-key block j < kAttnTraceBlocks, %globaltimer at [0] S_j seen by the softmax, [1] the row max
  // exchanged, [2] P_j written and announced, [3] the MMA warp's S_j issued
  unsigned long long* trace;
};
constexpr int kAttnTraceBlocks = 64;

constexpr int kAttnThreads = 256;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

constexpr int kAttnStages = 3;   // K/V tiles in flight per CTA

// Last CTA of a (group, row tile): merge the split-KV partial states (O unnormalised,
// m and l in the base-2 domain against any common reference).  (m, l) of every
// (split, row) go to shared memory in one coalesced pass, per-row weights
// w_s = 2^(m_s - M) / L are computed once, then every output element is reduced
// over the splits with independent loads spread over all threads.
template <int D>
__device__ __forceinline__ void combine_splits(const AttnArgs& a, size_t slot0, int tile, int b, int kvh,
                                               float* scratch, int tid, int nthreads) {
  const float kNegInf = __int_as_float(0xff800000);
  const int G = a.n_q / a.n_kv;
  const int rows_total = G * a.seq_q;
  const int nsplit = gridDim.z;
  float* sm_m = scratch;   // [nsplit][128]
  float* sm_l = sm_m + nsplit * 128;
  for (int i = tid; i < nsplit * 128; i += nthreads) {
    const float2 ml = __ldcg(&a.part_ml[slot0 * 128 + i]);
    sm_m[i] = ml.x;
    sm_l[i] = ml.y;
  }
  __syncthreads();
  if (tid < 128) {
    float mmax = kNegInf;
    for (int sp = 0; sp < nsplit; ++sp) mmax = fmaxf(mmax, sm_m[sp * 128 + tid]);
    float lsum = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) {
      const float w = exp2f(sm_m[sp * 128 + tid] - mmax);
      sm_m[sp * 128 + tid] = w;
      lsum += w * sm_l[sp * 128 + tid];
    }
    const float inv = 1.f / lsum;
    for (int sp = 0; sp < nsplit; ++sp) sm_m[sp * 128 + tid] *= inv;
  }
  __syncthreads();
  const int rows_here = min(128, rows_total - tile * 128);
  constexpr int Q4 = D / 4;
  constexpr int U = 8;   // output items per thread in flight
  const int total = rows_here * Q4;
  for (int base = tid; base < total; base += nthreads * U) {
    float4 o[U];
#pragma unroll
    for (int u = 0; u < U; ++u) o[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp = 0; sp < nsplit; ++sp) {
      float4 t[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int item = base + u * nthreads;
        if (item < total) {
          const int row = item / Q4, d4 = item - row * Q4;
          t[u] = __ldcg(reinterpret_cast<const float4*>(a.part_o + ((slot0 + sp) * 128 + row) * D) + d4);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int item = base + u * nthreads;
        if (item < total) {
          const float w = sm_m[sp * 128 + item / Q4];
          o[u].x += w * t[u].x;
          o[u].y += w * t[u].y;
          o[u].z += w * t[u].z;
          o[u].w += w * t[u].w;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int item = base + u * nthreads;
      if (item >= total) continue;
      const int row = item / Q4, d4 = item - row * Q4;
      const int pr = tile * 128 + row;
      const int head = kvh * G + pr / a.seq_q, pos = pr % a.seq_q;
      __nv_bfloat16* dst = a.o + ((static_cast<size_t>(b) * a.seq_q + pos) * a.n_q + head) * D + 4 * d4;
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(o[u].x, o[u].y), pack_bf16(o[u].z, o[u].w));
    }
  }
}

template <int D>
struct AttnSmem {
  static constexpr int kBytes = (128 + 2 * kAttnStages * 64) * D * 2;   // Q tile + K/V ring
};

template <int D>
__global__ void __launch_bounds__(kAttnThreads) attn_kernel(const AttnArgs a) {
  constexpr int CH = D / 8;                     // 16-byte chunks per row
  constexpr int SWM = CH >= 8 ? 7 : CH - 1;     // chunk swizzle mask
  const float kNegInf = __int_as_float(0xff800000);
  extern __shared__ __align__(128) uint8_t attn_smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(attn_smem);
  __nv_bfloat16* sK = sQ + 128 * D;
  __nv_bfloat16* sV = sK + kAttnStages * 64 * D;
  __shared__ int s_last;

  const int tile = blockIdx.x, grp = blockIdx.y, split = blockIdx.z;
  const int b = grp / a.n_kv, kvh = grp - b * a.n_kv;
  const int G = a.n_q / a.n_kv;
  const int rows_total = G * a.seq_q;
  const int total = a.len_a + a.len_b;
  const int nblk = (total + 63) >> 6;
  const int blk0 = split * a.blocks_per_split;
  const int blk1 = min(nblk, blk0 + a.blocks_per_split);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  auto off = [](int r, int c) { return r * D + ((c ^ (r & SWM)) << 3); };
  auto load_kv = [&](int blk, int buf) {
    for (int idx = tid; idx < 64 * CH; idx += kAttnThreads) {
      const int r = idx / CH, c = idx - (idx / CH) * CH;
      const int key = blk * 64 + r;
      const __nv_bfloat16 *ks = a.ka, *vs = a.va;
      const bool valid = key < total;
      if (key < a.len_a) {
        const size_t o = (static_cast<size_t>(grp) * a.len_a + key) * D + c * 8;
        ks = a.ka + o;
        vs = a.va + o;
      } else if (valid) {
        const size_t o = (static_cast<size_t>(grp) * a.len_b + (key - a.len_a)) * D + c * 8;
        ks = a.kb + o;
        vs = a.vb + o;
      }
      cp_async16(sK + buf * 64 * D + off(r, c), ks, valid);
      cp_async16(sV + buf * 64 * D + off(r, c), vs, valid);
    }
  };

  pdl_launch_dependents();
  // prologue: blocks blk0 .. blk0 + kAttnStages - 2 and the Q tile.  Commit groups are kept uniform:
  // group 0 = {block blk0 (+ any pre-issued blocks), Q}, then one group per further block.
  constexpr int NPRE = kAttnStages - 1;
  const bool pre = a.a_stable && (blk0 + NPRE) * 64 <= a.len_a && blk0 + NPRE <= blk1;
  if (pre)
    for (int i = 0; i < NPRE; ++i) load_kv(blk0 + i, i);   // the prefix cache predates the previous kernel
  pdl_wait();
  if (!pre && blk0 < blk1) load_kv(blk0, 0);
  for (int idx = tid; idx < 128 * CH; idx += kAttnThreads) {
    const int r = idx / CH, c = idx - (idx / CH) * CH;
    const int pr = tile * 128 + r;
    const bool valid = pr < rows_total;
    const __nv_bfloat16* src = a.q;
    if (valid) {
      const int head = kvh * G + pr / a.seq_q, pos = pr % a.seq_q;
      src = a.q + ((static_cast<size_t>(b) * a.seq_q + pos) * a.n_q + head) * D + c * 8;
    }
    cp_async16(sQ + off(r, c), src, valid);
  }
  cp_async_commit();
  for (int i = 1; i < NPRE; ++i) {
    if (!pre && blk0 + i < blk1) load_kv(blk0 + i, i);
    cp_async_commit();
  }

  float m_r[2] = {kNegInf, kNegInf}, l_r[2] = {0.f, 0.f};
  float acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  uint32_t qf[D / 16][4];
  const int g = lane >> 2, t4 = lane & 3;

  for (int blk = blk0; blk < blk1; ++blk) {
    const int it = blk - blk0;
    const int buf = it % kAttnStages;
    asm volatile("cp.async.wait_group %0;" ::"n"(kAttnStages - 2) : "memory");
    __syncthreads();
    if (it == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int row = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        ldsm_x4(qf[kk], smem_u32(sQ + off(row, kk * 2 + (lane >> 4))));
      }
    }
    // refill the slot computed on in the previous iteration (every thread passed the barrier above)
    if (blk + NPRE < blk1) load_kv(blk + NPRE, (it + NPRE) % kAttnStages);
    cp_async_commit();

    const __nv_bfloat16* Kb = sK + buf * 64 * D;
    const __nv_bfloat16* Vb = sV + buf * 64 * D;
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t bf[4];
        const int key = nt * 8 + (lane & 7) + 8 * (lane >> 4);
        ldsm_x4(bf, smem_u32(Kb + off(key, kk * 2 + ((lane >> 3) & 1))));
        mma_16816(s[nt], qf[kk], bf[0], bf[1]);
        mma_16816(s[nt + 1], qf[kk], bf[2], bf[3]);
      }
    }
    // mask keys past the end, then the online-softmax update for rows g and g + 8
    const int kbase = blk * 64;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int key = kbase + nt * 8 + 2 * t4 + (j & 1);
        s[nt][j] = key < total ? s[nt][j] * a.scale_log2 : kNegInf;
      }
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      float mx = kNegInf;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * h2], s[nt][2 * h2 + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_r[h2], mx);
      const float alpha = exp2f(m_r[h2] - m_new);
      m_r[h2] = m_new;
      float sum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s[nt][2 * h2] = exp2f(s[nt][2 * h2] - m_new);
        s[nt][2 * h2 + 1] = exp2f(s[nt][2 * h2 + 1] - m_new);
        sum += s[nt][2 * h2] + s[nt][2 * h2 + 1];
      }
      l_r[h2] = l_r[h2] * alpha + sum;
#pragma unroll
      for (int dt = 0; dt < D / 8; ++dt) {
        acc[dt][2 * h2] *= alpha;
        acc[dt][2 * h2 + 1] *= alpha;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dt = 0; dt < D / 8; dt += 2) {
        uint32_t bf[4];
        const int key = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        ldsm_x4_t(bf, smem_u32(Vb + off(key, dt + (lane >> 4))));
        mma_16816(acc[dt], pa, bf[0], bf[1]);
        mma_16816(acc[dt + 1], pa, bf[2], bf[3]);
      }
    }
  }
  cp_async_wait_all();
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    l_r[h2] += __shfl_xor_sync(0xffffffffu, l_r[h2], 1);
    l_r[h2] += __shfl_xor_sync(0xffffffffu, l_r[h2], 2);
  }

  if (gridDim.z == 1) {
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int pr = tile * 128 + warp * 16 + g + 8 * h2;
      if (pr >= rows_total) continue;
      const int head = kvh * G + pr / a.seq_q, pos = pr % a.seq_q;
      __nv_bfloat16* dst = a.o + ((static_cast<size_t>(b) * a.seq_q + pos) * a.n_q + head) * D;
      const float inv = 1.f / l_r[h2];
#pragma unroll
      for (int dt = 0; dt < D / 8; ++dt) {
        const int d = dt * 8 + 2 * t4;
        *reinterpret_cast<__nv_bfloat162*>(dst + d) =
            __floats2bfloat162_rn(acc[dt][2 * h2] * inv, acc[dt][2 * h2 + 1] * inv);
      }
    }
    return;
  }

  // ---- split keys: publish the partial state, the last CTA of the group combines
  const size_t slot0 = (static_cast<size_t>(grp) * gridDim.x + tile) * gridDim.z;
  const size_t mine = (slot0 + split) * 128;
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int row = warp * 16 + g + 8 * h2;
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) {
      const int d = dt * 8 + 2 * t4;
      *reinterpret_cast<float2*>(a.part_o + (mine + row) * D + d) = make_float2(acc[dt][2 * h2], acc[dt][2 * h2 + 1]);
    }
    if (t4 == 0) a.part_ml[mine + row] = make_float2(m_r[h2], l_r[h2]);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    int* ctr = a.counters + static_cast<size_t>(grp) * gridDim.x + tile;
    const int prev = atomicAdd(ctr, 1);
    s_last = prev == static_cast<int>(gridDim.z) - 1;
    if (s_last) *ctr = 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  combine_splits<D>(a, slot0, tile, b, kvh, reinterpret_cast<float*>(attn_smem), tid, kAttnThreads);
}

}  // namespace dm0
