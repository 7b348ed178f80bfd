// One flow-matching training step of the action expert (DM0.5 page, section 5.3: x_t = t eps + (1 - t) a,
// u_t = eps - a, the masked mean squared error between v(x_t, t | c) and u_t; DM0 architecture notes,
// section 1: knowledge insulation keeps the prefix K/V a constant).  The dense contractions (forward
// projections, dX = dY W and dW = dY^T X of every projection) run on the tcgen05 GEMM with both
// operands K-major: dX uses transposed weight copies, dW the token-padded transposes of dY and X.
// The kernels here are the rest, on CUDA cores: the input and the head with the loss, RMSNorm forward
// and backward, QK-norm + RoPE forward and backward, SwiGLU forward and backward, the merged
// attention over [prefix cache; suffix] forward (probabilities kept) and backward, transposes and
// token reductions.  Layouts: tokens t = b S + s; activations [T][features] fp32 unless noted.
#pragma once
#include "ptx.cuh"

namespace dm0 {

// number of valid entries of the mask (count zeroed by the caller)
__global__ void __launch_bounds__(256) train_count_kernel(const uint8_t* mask, int n, int* count) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int red[8];
  int c = 0;
  for (int i = blockIdx.x * 256 + threadIdx.x; i < n; i += gridDim.x * 256) c += mask[i] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int w = 0; w < 8; ++w) tot += red[w];
    atomicAdd(count, tot);
  }
}

// per token (one CTA): x_t = t eps + (1 - t) a and u = eps - a of its sample's t, and the expert's input
// e = x_t W_in^T + b_in + tau(t) (tau as in the Euler loop's step kernel)
__global__ void __launch_bounds__(256) train_input_kernel(const float* a, const float* eps, const float* t,
                                                          const __nv_bfloat16* W_in, const float* b_in, int S, int A,
                                                          int Ha, float* xt, float* u, float* h) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float sx[64];
  const int tok = blockIdx.x, b = tok / S;
  const float tb = t[b];
  for (int i = threadIdx.x; i < A; i += blockDim.x) {
    const size_t k = static_cast<size_t>(tok) * A + i;
    const float e = eps[k], av = a[k];
    const float x = tb * e + (1.f - tb) * av;
    sx[i] = x;
    xt[k] = x;
    u[k] = e - av;
  }
  __syncthreads();
  const int half = Ha >> 1;
  const float kLog2_10000 = 13.287712379549449f;
  for (int j = threadIdx.x; j < Ha; j += blockDim.x) {
    float e = b_in[j];
    const __nv_bfloat16* w = W_in + static_cast<size_t>(j) * A;
    for (int i = 0; i < A; ++i) e += __bfloat162float(w[i]) * sx[i];
    const int fi = j < half ? j : j - half;
    const float arg = tb * exp2f(-static_cast<float>(fi) / half * kLog2_10000);
    e += j < half ? sinf(arg) : cosf(arg);
    h[static_cast<size_t>(tok) * Ha + j] = e;
  }
}

// RMSNorm of rows (one warp per row): rho = 1 / sqrt(mean(x^2) + eps), out = bf16(x rho g) (a GEMM operand)
__global__ void __launch_bounds__(256) train_rms_kernel(const float* x, const float* g, int rows, int H, float eps,
                                                        __nv_bfloat16* out, float* rho) {
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* xr = x + static_cast<size_t>(row) * H;
  float ss = 0.f;
  for (int j = lane; j < H; j += 32) ss += xr[j] * xr[j];
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / H + eps);
  if (lane == 0) rho[row] = r;
  for (int j = lane; j < H; j += 32) out[static_cast<size_t>(row) * H + j] = __float2bfloat16_rn(xr[j] * r * g[j]);
}

// adjoint of y = g n, n = x rho (one warp per row): dx = dres + rho (dn - n mean(dn n)), dn = g dy
__global__ void __launch_bounds__(256) train_rms_bwd_kernel(const float* dy, const float* x, const float* g,
                                                            const float* rho, const float* dres, int rows, int H,
                                                            float* dx) {
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const size_t o = static_cast<size_t>(row) * H;
  const float r = rho[row];
  float m = 0.f;
  for (int j = lane; j < H; j += 32) m += g[j] * dy[o + j] * x[o + j] * r;
  m = warp_sum(m) / H;
  for (int j = lane; j < H; j += 32) dx[o + j] = dres[o + j] + r * (g[j] * dy[o + j] - x[o + j] * r * m);
}

// dg[j] = sum over rows of dy[t][j] x[t][j] rho[t] (the gain's gradient; one thread per column)
__global__ void __launch_bounds__(256) train_gain_grad_kernel(const float* dy, const float* x, const float* rho,
                                                              int rows, int H, float* dg) {
  pdl_launch_dependents();
  pdl_wait();
  const int j = blockIdx.x * 256 + threadIdx.x;
  if (j >= H) return;
  float acc = 0.f;
  for (int t = 0; t < rows; ++t) acc += dy[static_cast<size_t>(t) * H + j] * x[static_cast<size_t>(t) * H + j] * rho[t];
  dg[j] = acc;
}

// out[p][q] = sum over rows of L[t][p] R[t][q] (the small outer-product gradients dW_in, dW_out;
// one thread per output), and colsum[p] = sum over rows of L[t][p] when colsum is not null
__global__ void __launch_bounds__(256) train_outer_kernel(const float* L, const float* R, int rows, int NP, int NQ,
                                                          float* out, float* colsum) {
  pdl_launch_dependents();
  pdl_wait();
  const int idx = blockIdx.x * 256 + threadIdx.x;
  if (idx >= NP * NQ) return;
  const int p = idx / NQ, q = idx - (idx / NQ) * NQ;
  float acc = 0.f, cs = 0.f;
  for (int t = 0; t < rows; ++t) {
    const float l = L[static_cast<size_t>(t) * NP + p];
    acc += l * R[static_cast<size_t>(t) * NQ + q];
    cs += l;
  }
  out[idx] = acc;
  if (colsum && q == 0) colsum[p] = cs;
}

// h_out = h_in + y (the residual add after a projection computed by a StoreF32 GEMM)
__global__ void __launch_bounds__(256) train_add_kernel(const float* h_in, const float* y, size_t n, float* h_out) {
  pdl_launch_dependents();
  pdl_wait();
  for (size_t i = blockIdx.x * 256ull + threadIdx.x; i < n; i += static_cast<size_t>(gridDim.x) * 256) h_out[i] = h_in[i] + y[i];
}

// fp32 or bf16 [R][C] -> bf16 [C][Rp] (rows R..Rp-1 of the output are zero): the K-major operands of a
// dW = dY^T X GEMM (tokens along K) and the transposed weight copies.  32 x 32 tiles through shared memory.
template <typename Tin>
__global__ void __launch_bounds__(256) train_transpose_kernel(const Tin* src, int R, int C, int Rp, __nv_bfloat16* dst) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const int r = r0 + i, cc = c0 + tx;
    float v = 0.f;
    if (r < R && cc < C) {
      if constexpr (sizeof(Tin) == 2)
        v = __bfloat162float(src[static_cast<size_t>(r) * C + cc]);
      else
        v = src[static_cast<size_t>(r) * C + cc];
    }
    tile[i][tx] = v;
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int cc = c0 + i, r = r0 + tx;
    if (cc < C && r < Rp) dst[static_cast<size_t>(cc) * Rp + r] = __float2bfloat16_rn(tile[tx][i]);
  }
}

// fp32 -> bf16 copy (the dY operands of dX = dY W)
__global__ void __launch_bounds__(256) train_to_bf16_kernel(const float* x, size_t n, __nv_bfloat16* y) {
  pdl_launch_dependents();
  pdl_wait();
  for (size_t i = blockIdx.x * 256ull + threadIdx.x; i < n; i += static_cast<size_t>(gridDim.x) * 256)
    y[i] = __float2bfloat16_rn(x[i]);
}

// QK-norm + RoPE of the suffix's own q and k (one warp per (token, head) of the n_q + n_kv q/k heads):
// from the raw projections raw [T][QR] (q heads, then k heads, then v heads), keep per head rho and
// the rotated result in fp32; v is copied.  Positions P + s.
__global__ void __launch_bounds__(256) train_qk_fwd_kernel(const float* raw, const float* qg, const float* kg,
                                                           const float2* rope, int T, int S, int P, int Hq, int Hkv,
                                                           int D, float eps, float* qr, float* kr, float* v,
                                                           float* rho_q, float* rho_k) {
  pdl_launch_dependents();
  pdl_wait();
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const int heads = Hq + 2 * Hkv;
  if (w >= T * heads) return;
  const int tok = w / heads, hh = w - tok * heads;
  const int QR = heads * D, half = D >> 1;
  const float* x = raw + static_cast<size_t>(tok) * QR + hh * D;
  if (hh >= Hq + Hkv) {   // v head
    const int g = hh - Hq - Hkv;
    for (int d = lane; d < D; d += 32) v[(static_cast<size_t>(tok) * Hkv + g) * D + d] = x[d];
    return;
  }
  const bool isq = hh < Hq;
  const float* gain = isq ? qg : kg;
  float ss = 0.f;
  for (int d = lane; d < D; d += 32) ss += x[d] * x[d];
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / D + eps);
  const int pos = P + tok % S;
  float* out = isq ? qr + (static_cast<size_t>(tok) * Hq + hh) * D : kr + (static_cast<size_t>(tok) * Hkv + hh - Hq) * D;
  if (lane == 0) {
    if (isq)
      rho_q[static_cast<size_t>(tok) * Hq + hh] = r;
    else
      rho_k[static_cast<size_t>(tok) * Hkv + hh - Hq] = r;
  }
  for (int i = lane; i < half; i += 32) {
    const float2 cs = rope[static_cast<size_t>(pos) * half + i];
    const float x0 = x[i] * r * gain[i], x1 = x[i + half] * r * gain[i + half];
    out[i] = x0 * cs.x - x1 * cs.y;
    out[i + half] = x1 * cs.x + x0 * cs.y;
  }
}

// adjoint of train_qk_fwd for the q and k heads (one warp per (token, head)): the rotation transposed,
// then the RMSNorm adjoint; writes bf16 d(raw) of q / k heads into dqkv and the suffix rows of dV into
// its v heads; the gains' gradients are added atomically.  dK / dV rows of the suffix are at P + s of
// the sample's [P + S] keys.
__global__ void __launch_bounds__(256) train_qk_bwd_kernel(const float* raw, const float* qg, const float* kg,
                                                           const float2* rope, const float* rho_q, const float* rho_k,
                                                           const float* dqr, const float* dK, const float* dV, int T,
                                                           int S, int P, int Hq, int Hkv, int D, __nv_bfloat16* dqkv,
                                                           float* dgq, float* dgk) {
  pdl_launch_dependents();
  pdl_wait();
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const int heads = Hq + 2 * Hkv;
  if (w >= T * heads) return;
  const int tok = w / heads, hh = w - tok * heads;
  const int QR = heads * D, half = D >> 1, b = tok / S, s = tok - (tok / S) * S;
  const float* x = raw + static_cast<size_t>(tok) * QR + hh * D;
  __nv_bfloat16* dx = dqkv + static_cast<size_t>(tok) * QR + hh * D;
  if (hh >= Hq + Hkv) {   // v head: dV of the suffix key
    const int g = hh - Hq - Hkv;
    const float* src = dV + ((static_cast<size_t>(b) * Hkv + g) * (P + S) + P + s) * D;
    for (int d = lane; d < D; d += 32) dx[d] = __float2bfloat16_rn(src[d]);
    return;
  }
  const bool isq = hh < Hq;
  const float* gain = isq ? qg : kg;
  float* dg = isq ? dgq : dgk;
  const float r = isq ? rho_q[static_cast<size_t>(tok) * Hq + hh] : rho_k[static_cast<size_t>(tok) * Hkv + hh - Hq];
  const float* dy = isq ? dqr + (static_cast<size_t>(tok) * Hq + hh) * D
                        : dK + ((static_cast<size_t>(b) * Hkv + (hh - Hq)) * (P + S) + P + s) * D;
  const int pos = P + s;
  // pass 1: m = mean(dn n) with dn = g R^T dy, n = x rho
  float m = 0.f;
  for (int i = lane; i < half; i += 32) {
    const float2 cs = rope[static_cast<size_t>(pos) * half + i];
    const float d0 = dy[i] * cs.x + dy[i + half] * cs.y, d1 = dy[i + half] * cs.x - dy[i] * cs.y;
    m += gain[i] * d0 * x[i] * r + gain[i + half] * d1 * x[i + half] * r;
  }
  m = warp_sum(m) / D;
  for (int i = lane; i < half; i += 32) {
    const float2 cs = rope[static_cast<size_t>(pos) * half + i];
    const float d0 = dy[i] * cs.x + dy[i + half] * cs.y, d1 = dy[i + half] * cs.x - dy[i] * cs.y;
    const float n0 = x[i] * r, n1 = x[i + half] * r;
    dx[i] = __float2bfloat16_rn(r * (gain[i] * d0 - n0 * m));
    dx[i + half] = __float2bfloat16_rn(r * (gain[i + half] * d1 - n1 * m));
    atomicAdd(dg + i, d0 * n0);
    atomicAdd(dg + i + half, d1 * n1);
  }
}

// SwiGLU forward from the interleaved gate/up projection gu [T][2I] (rows [128j, 128j+64) gate block j,
// [128j+64, 128j+128) up block j): act[t][i] = bf16(silu(gate) up)
__global__ void __launch_bounds__(256) train_swiglu_kernel(const float* gu, int T, int I, __nv_bfloat16* act) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t n = static_cast<size_t>(T) * I;
  for (size_t k = blockIdx.x * 256ull + threadIdx.x; k < n; k += static_cast<size_t>(gridDim.x) * 256) {
    const size_t tok = k / I;
    const int i = static_cast<int>(k - tok * I), blk = i >> 6, w = i & 63;
    const float g = gu[tok * 2 * I + 128 * blk + w], u = gu[tok * 2 * I + 128 * blk + 64 + w];
    act[k] = __float2bfloat16_rn(g / (1.f + expf(-g)) * u);
  }
}

// its adjoint: dgate = dact up sigma(g) (1 + g (1 - sigma(g))), dup = dact silu(g), interleaved as gu
__global__ void __launch_bounds__(256) train_swiglu_bwd_kernel(const float* gu, const float* dact, int T, int I,
                                                               __nv_bfloat16* dgu) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t n = static_cast<size_t>(T) * I;
  for (size_t k = blockIdx.x * 256ull + threadIdx.x; k < n; k += static_cast<size_t>(gridDim.x) * 256) {
    const size_t tok = k / I;
    const int i = static_cast<int>(k - tok * I), blk = i >> 6, w = i & 63;
    const size_t gi = tok * 2 * I + 128 * blk + w, ui = gi + 64;
    const float g = gu[gi], u = gu[ui], da = dact[k];
    const float sg = 1.f / (1.f + expf(-g));
    dgu[gi] = __float2bfloat16_rn(da * u * sg * (1.f + g * (1.f - sg)));
    dgu[ui] = __float2bfloat16_rn(da * g * sg);
  }
}

// gradient of the interleaved gate/up weight [2I][H] into the separate Wg, Wu [I][H] slots
__global__ void __launch_bounds__(256) train_deinterleave_kernel(const float* dgu, int I, int H, float* dWg, float* dWu) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t n = static_cast<size_t>(2 * I) * H;
  for (size_t k = blockIdx.x * 256ull + threadIdx.x; k < n; k += static_cast<size_t>(gridDim.x) * 256) {
    const size_t row = k / H, col = k - row * H;
    const int blk = static_cast<int>(row >> 7), w = static_cast<int>(row & 127);
    const size_t out = (static_cast<size_t>(blk) * 64 + (w & 63)) * H + col;
    (w < 64 ? dWg : dWu)[out] = dgu[k];
  }
}

// Merged attention of the training step on CUDA cores, for head_dim 32 and 64 (head_dim 128 runs the
// tcgen05 flash attention and its adjoint kernel): one CTA per (sample, query head), all S query rows: scores
// against the sample's [prefix cache (bf16); suffix keys (fp32)] keys, softmax (fp32), probabilities
// kept in prob [B][Hq][S][P + S], o = prob V in fp32 and bf16.  Shared memory: q [S][D], a 32-key
// tile [32][D + 1], a probability tile [S][32].
struct TrainAttn {
  const float *qr, *kr, *vs;          // [T][Hq D], [T][Hkv D], [T][Hkv D]
  const __nv_bfloat16 *kc, *vc;       // [B][Hkv][P][D] prefix cache
  int B, S, P, Hq, Hkv, D;
  float scale;
  float* prob;                        // [B][Hq][S][P + S]
  float* of;                          // [T][Hq D]
  __nv_bfloat16* of_bf;
  // backward
  const float* dof;                   // [T][Hq D]
  float* dqr;                         // [T][Hq D]
  float *dK, *dV;                     // [B][Hkv][P + S][D], accumulated (zeroed by the caller)
};

// key / value tiles are [32][D + 1]: the padding puts the 32 keys a warp reads at one dimension in 32
// different banks
__device__ __forceinline__ void train_load_keys(const TrainAttn& a, bool values, int b, int g, int k0, float* tile) {
  const int N = a.P + a.S, KP = a.D + 1;
  for (int idx = threadIdx.x; idx < 32 * a.D; idx += blockDim.x) {
    const int kk = idx / a.D, d = idx - (idx / a.D) * a.D, k = k0 + kk;
    float v = 0.f;
    if (k < a.P)
      v = __bfloat162float((values ? a.vc : a.kc)[((static_cast<size_t>(b) * a.Hkv + g) * a.P + k) * a.D + d]);
    else if (k < N)
      v = (values ? a.vs : a.kr)[(static_cast<size_t>(b * a.S + k - a.P) * a.Hkv + g) * a.D + d];
    tile[kk * KP + d] = v;
  }
}

__global__ void __launch_bounds__(256) train_attn_fwd_kernel(const TrainAttn a) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ float sm[];
  const int b = blockIdx.x / a.Hq, h = blockIdx.x - (blockIdx.x / a.Hq) * a.Hq, g = h / (a.Hq / a.Hkv);
  const int S = a.S, D = a.D, N = a.P + a.S, KP = D + 1;
  float* sq = sm;                // [S][D]
  float* st = sq + S * D;        // [32][D + 1]
  float* sp = st + 32 * KP;      // [S][32]
  float* prob = a.prob + (static_cast<size_t>(b) * a.Hq + h) * S * N;
  for (int idx = threadIdx.x; idx < S * D; idx += blockDim.x) {
    const int s = idx / D, d = idx - (idx / D) * D;
    sq[idx] = a.qr[(static_cast<size_t>(b * S + s) * a.Hq + h) * D + d];
  }
  // scores
  for (int k0 = 0; k0 < N; k0 += 32) {
    __syncthreads();
    train_load_keys(a, false, b, g, k0, st);
    __syncthreads();
    for (int idx = threadIdx.x; idx < S * 32; idx += blockDim.x) {
      const int s = idx >> 5, kk = idx & 31;
      if (k0 + kk >= N) continue;
      float acc = 0.f;
      for (int d = 0; d < D; ++d) acc += sq[s * D + d] * st[kk * KP + d];
      prob[static_cast<size_t>(s) * N + k0 + kk] = acc * a.scale;
    }
  }
  __syncthreads();
  // softmax per row (one warp per row)
  for (int s = threadIdx.x >> 5; s < S; s += blockDim.x >> 5) {
    float* row = prob + static_cast<size_t>(s) * N;
    const int lane = threadIdx.x & 31;
    float mx = -INFINITY;
    for (int k = lane; k < N; k += 32) mx = fmaxf(mx, row[k]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int k = lane; k < N; k += 32) {
      const float e = expf(row[k] - mx);
      row[k] = e;
      sum += e;
    }
    sum = warp_sum(sum);
    const float inv = 1.f / sum;
    for (int k = lane; k < N; k += 32) row[k] *= inv;
  }
  __syncthreads();
  // o = prob V: each thread owns outputs (s, d) = idx, idx + 256, ...
  constexpr int kMaxOut = 32;
  float acc[kMaxOut];
#pragma unroll
  for (int i = 0; i < kMaxOut; ++i) acc[i] = 0.f;
  for (int k0 = 0; k0 < N; k0 += 32) {
    __syncthreads();
    train_load_keys(a, true, b, g, k0, st);
    for (int idx = threadIdx.x; idx < S * 32; idx += blockDim.x) {
      const int s = idx >> 5, kk = idx & 31;
      sp[idx] = k0 + kk < N ? prob[static_cast<size_t>(s) * N + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kMaxOut; ++i) {
      const int idx = threadIdx.x + i * blockDim.x;
      if (idx >= S * D) break;
      const int s = idx / D, d = idx - (idx / D) * D;
      float v = 0.f;
      for (int kk = 0; kk < 32; ++kk) v += sp[s * 32 + kk] * st[kk * KP + d];
      acc[i] += v;
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxOut; ++i) {
    const int idx = threadIdx.x + i * blockDim.x;
    if (idx >= S * D) break;
    const int s = idx / D, d = idx - (idx / D) * D;
    const size_t o = (static_cast<size_t>(b * S + s) * a.Hq + h) * D + d;
    a.of[o] = acc[i];
    a.of_bf[o] = __float2bfloat16_rn(acc[i]);
  }
}

// Backward of train_attn_fwd, one CTA per (sample, query head): delta_s = sum_d dO O;
// dS = prob (dO V^T - delta) scale; dq = dS K; dK += dS^T q; dV += prob^T dO (atomically: the query
// heads of a group share their KV head).  Shared memory: q, dO [S][D], K and V tiles [32][D + 1], the
// dS and probability tiles [S][32], delta [S].
__global__ void __launch_bounds__(256) train_attn_bwd_kernel(const TrainAttn a) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ float sm[];
  const int b = blockIdx.x / a.Hq, h = blockIdx.x - (blockIdx.x / a.Hq) * a.Hq, g = h / (a.Hq / a.Hkv);
  const int S = a.S, D = a.D, N = a.P + a.S, KP = D + 1;
  float* sq = sm;                 // [S][D]
  float* sdo = sq + S * D;        // [S][D]
  float* sk = sdo + S * D;        // [32][D + 1]
  float* sv = sk + 32 * KP;       // [32][D + 1]
  float* sds = sv + 32 * KP;      // [S][32]
  float* sp = sds + S * 32;       // [S][32]
  float* sdelta = sp + S * 32;    // [S]
  const float* prob = a.prob + (static_cast<size_t>(b) * a.Hq + h) * S * N;
  for (int idx = threadIdx.x; idx < S * D; idx += blockDim.x) {
    const int s = idx / D, d = idx - (idx / D) * D;
    const size_t o = (static_cast<size_t>(b * S + s) * a.Hq + h) * D + d;
    sq[idx] = a.qr[o];
    sdo[idx] = a.dof[o];
  }
  __syncthreads();
  for (int s = threadIdx.x >> 5; s < S; s += blockDim.x >> 5) {
    const int lane = threadIdx.x & 31;
    float dl = 0.f;
    for (int d = lane; d < D; d += 32) dl += sdo[s * D + d] * a.of[(static_cast<size_t>(b * S + s) * a.Hq + h) * D + d];
    dl = warp_sum(dl);
    if (lane == 0) sdelta[s] = dl;
  }
  constexpr int kMaxOut = 32;
  float dq[kMaxOut];
#pragma unroll
  for (int i = 0; i < kMaxOut; ++i) dq[i] = 0.f;
  float* dK = a.dK + (static_cast<size_t>(b) * a.Hkv + g) * N * D;
  float* dV = a.dV + (static_cast<size_t>(b) * a.Hkv + g) * N * D;
  for (int k0 = 0; k0 < N; k0 += 32) {
    __syncthreads();
    train_load_keys(a, false, b, g, k0, sk);
    train_load_keys(a, true, b, g, k0, sv);
    __syncthreads();
    for (int idx = threadIdx.x; idx < S * 32; idx += blockDim.x) {
      const int s = idx >> 5, kk = idx & 31;
      float p = 0.f, ds = 0.f;
      if (k0 + kk < N) {
        p = prob[static_cast<size_t>(s) * N + k0 + kk];
        float dp = 0.f;
        for (int d = 0; d < D; ++d) dp += sdo[s * D + d] * sv[kk * KP + d];
        ds = p * (dp - sdelta[s]) * a.scale;
      }
      sp[idx] = p;
      sds[idx] = ds;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kMaxOut; ++i) {
      const int idx = threadIdx.x + i * blockDim.x;
      if (idx >= S * D) break;
      const int s = idx / D, d = idx - (idx / D) * D;
      float v = 0.f;
      for (int kk = 0; kk < 32; ++kk) v += sds[s * 32 + kk] * sk[kk * KP + d];
      dq[i] += v;
    }
    for (int idx = threadIdx.x; idx < 32 * D; idx += blockDim.x) {
      const int kk = idx / D, d = idx - (idx / D) * D;
      if (k0 + kk >= N) continue;
      float vk = 0.f, vv = 0.f;
      for (int s = 0; s < S; ++s) {
        vk += sds[s * 32 + kk] * sq[s * D + d];
        vv += sp[s * 32 + kk] * sdo[s * D + d];
      }
      atomicAdd(dK + static_cast<size_t>(k0 + kk) * D + d, vk);
      atomicAdd(dV + static_cast<size_t>(k0 + kk) * D + d, vv);
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxOut; ++i) {
    const int idx = threadIdx.x + i * blockDim.x;
    if (idx >= S * D) break;
    const int s = idx / D, d = idx - (idx / D) * D;
    a.dqr[(static_cast<size_t>(b * S + s) * a.Hq + h) * D + d] = dq[i];
  }
}

// Operands of the training step's tensor-core attention from the fp32 layer intermediates: q (after
// QK-norm and RoPE) in bf16 in its own layout [T][Hq D], and the suffix keys and values in bf16 as the
// second key segment [B][Hkv][S][D] (the prefix cache is the first).  One thread per element.
__global__ void __launch_bounds__(256) train_attn_prep_kernel(const float* qr, const float* kr, const float* vs, int B,
                                                              int S, int Hq, int Hkv, int D, __nv_bfloat16* q_bf,
                                                              __nv_bfloat16* k_bf, __nv_bfloat16* v_bf) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t nq = static_cast<size_t>(B) * S * Hq * D, nk = static_cast<size_t>(B) * S * Hkv * D;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < nq + nk; i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    if (i < nq) {
      q_bf[i] = __float2bfloat16_rn(qr[i]);
      continue;
    }
    const size_t k = i - nq;   // source [b S + s][g D + d] -> [b][g][s][d]
    const int d = static_cast<int>(k % D);
    const size_t rest = k / D;
    const int g = static_cast<int>(rest % Hkv);
    const size_t t = rest / Hkv;
    const int b = static_cast<int>(t / S), s = static_cast<int>(t % S);
    const size_t dst = ((static_cast<size_t>(b) * Hkv + g) * S + s) * D + d;
    k_bf[dst] = __float2bfloat16_rn(kr[k]);
    v_bf[dst] = __float2bfloat16_rn(vs[k]);
  }
}

// The head of the step, one CTA per token: rf = RMSNorm_final(h_L), v = rf W_out^T + b_out, the masked
// squared error against u added to loss (divided by the valid count), dv = 2 m (v - u) / N, and the
// adjoint back to dh (the final norm's input); rf, dv and drf are kept for the weight gradients.
__global__ void __launch_bounds__(256) train_head_kernel(const float* h, const float* fnorm, const __nv_bfloat16* W_out,
                                                         const float* b_out, const float* u, const uint8_t* mask,
                                                         const int* count, int Ha, int A, float eps, float* rf,
                                                         float* rho, float* dv, float* drf, float* dh, float* loss) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ float hs[];   // [Ha] rf, then [Ha] drf
  __shared__ float sdv[64];
  __shared__ float red[8];
  const int tok = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* hr = h + static_cast<size_t>(tok) * Ha;
  float ss = 0.f;
  for (int j = threadIdx.x; j < Ha; j += 256) ss += hr[j] * hr[j];
  ss = warp_sum(ss);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < 8; ++w) tot += red[w];
  const float r = rsqrtf(tot / Ha + eps);
  for (int j = threadIdx.x; j < Ha; j += 256) {
    hs[j] = hr[j] * r * fnorm[j];
    rf[static_cast<size_t>(tok) * Ha + j] = hs[j];
  }
  if (threadIdx.x == 0) rho[tok] = r;
  __syncthreads();
  const float inv_n = 1.f / static_cast<float>(max(*count, 1));
  float lsum = 0.f;
  for (int o = warp; o < A; o += 8) {
    const __nv_bfloat16* wr = W_out + static_cast<size_t>(o) * Ha;
    float acc = 0.f;
    for (int j = lane; j < Ha; j += 32) acc += __bfloat162float(wr[j]) * hs[j];
    acc = warp_sum(acc);
    if (lane == 0) {
      const size_t k = static_cast<size_t>(tok) * A + o;
      const float diff = mask[k] ? acc + b_out[o] - u[k] : 0.f;
      lsum += diff * diff;
      const float d = 2.f * diff * inv_n;
      sdv[o] = d;
      dv[k] = d;
    }
  }
  __syncthreads();
  if (lane == 0) red[warp] = lsum;
  __syncthreads();
  if (threadIdx.x == 0) {
    float l = 0.f;
    for (int w = 0; w < 8; ++w) l += red[w];
    atomicAdd(loss, l * inv_n);
  }
  float* sdr = hs + Ha;
  float m = 0.f;
  for (int j = threadIdx.x; j < Ha; j += 256) {
    float d = 0.f;
    for (int o = 0; o < A; ++o) d += sdv[o] * __bfloat162float(W_out[static_cast<size_t>(o) * Ha + j]);
    sdr[j] = d;
    drf[static_cast<size_t>(tok) * Ha + j] = d;
    m += fnorm[j] * d * hr[j] * r;
  }
  m = warp_sum(m);
  __syncthreads();
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float mt = 0.f;
  for (int w = 0; w < 8; ++w) mt += red[w];
  mt /= Ha;
  for (int j = threadIdx.x; j < Ha; j += 256)
    dh[static_cast<size_t>(tok) * Ha + j] = r * (fnorm[j] * sdr[j] - hr[j] * r * mt);
}

}  // namespace dm0
