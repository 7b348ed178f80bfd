// Small bandwidth-trivial kernels around the GEMM/attention chain:
//   rows_prep    : residual stream in (bf16 prefix embeddings or fp32), first
//                  pending RMSNorm operand bf16(g * h) and its sum of squares.
//   step_kernel  : per action token, the flow-matching step boundary
//                  (DM0.5 page, sections 5.2-5.3): velocity
//                  v = RMSNorm_final(h) W_out^T + b_out, Euler update
//                  x <- x + dt v with dt = -1/K, then the next step's input
//                  e = x W_in^T + b_in + tau(t) with t = 1 - k/K.
//   rope_table   : (cos, sin) of position * theta^(-2i/D), in double precision.
//   tmod_*       : the time-modulation tables of the time-modulated action expert.
//   quant_rows_e4m3 : per-row FP8 E4M3 codes and scales.
#pragma once
#include <cuda_fp8.h>

#include "ptx.cuh"

namespace dm0 {

// h[row] = in[row]; xn[row] = bf16(gain * h); ssq[0][row] = sum h^2; ssq[s][row] = 0 for s >= 1
// (the n_slots partial-sum slots a consumer adds up).  One warp per row.
__global__ void __launch_bounds__(256) rows_prep_kernel(const void* in, int in_bf16, float* h, __nv_bfloat16* xn,
                                                        const float* gain, float* ssq, int n_slots, int slot_stride,
                                                        int M, int H) {
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= M) return;
  float sq = 0.f;
  for (int c = lane; c < H; c += 32) {
    const size_t i = static_cast<size_t>(row) * H + c;
    const float v = in_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(in)[i])
                            : reinterpret_cast<const float*>(in)[i];
    h[i] = v;
    xn[i] = __float2bfloat16_rn(gain[c] * v);
    sq += v * v;
  }
  sq = warp_sum(sq);
  if (lane == 0) {
    ssq[row] = sq;
    for (int s = 1; s < n_slots; ++s) ssq[static_cast<size_t>(s) * slot_stride + row] = 0.f;
  }
}

struct StepArgs {
  float* x;                    // [tokens][A] flow state
  float* h;                    // action residual stream: element (token, j) at h[token * h_ts + j * h_fs]
  int h_ts, h_fs;              // [tokens][Ha] row-major: (Ha, 1); feature-major [Ha][64]: (1, 64)
  __nv_bfloat16* xn;           // [tokens][Ha] bf16(attn_norm_0 * h)
  float* ssq;                  // [n_slots][tokens]
  int n_slots, tokens;
  const __nv_bfloat16* W_in;   // [Ha][A]
  const float* b_in;           // [Ha]
  const float* attn_norm0;     // [Ha] gain of the first action layer's input norm
  const float* final_norm;     // [Ha]
  const __nv_bfloat16* W_out;  // [A][Ha]
  const float* b_out;          // [A]
  int Ha, A;
  float eps;
  int k_out;                   // step whose velocity is applied (-1: none)
  int k_in;                    // step whose input is built (-1: none)
  int steps;
  float* vel;                  // [steps][tokens][A] or null
};

// Step boundary for one action token, run by `nthr` threads (a multiple of 32, >= the action
// dimension, <= 256) that synchronise with `sync()`.  `hs` is shared scratch for Ha floats.  Reads
// of h go through L2: in the persistent Euler loop other CTAs produced them.  xn / ssq are written
// only when non-null.  Weight rows are read 16 bytes at a time when the shapes allow it, so the
// loads of a row are in flight together.
// kMod: the time-modulated expert's step: final_norm holds the final norm's 1 + scale, final_shift
// ([Ha]) its shift, and the time embedding is not added to the input (time enters through the
// modulators).  kMod = false compiles the DM0 step (final_shift unused).
template <bool kMod = false, class Sync>
__device__ __forceinline__ void step_token(const StepArgs& a, int tok, int tid, int nthr, float* sx, float* sred,
                                           float* hs, Sync&& sync, const float* final_shift = nullptr) {
  const int nw = nthr >> 5, warp = tid >> 5, lane = tid & 31;
  float* hrow = a.h + static_cast<size_t>(tok) * a.h_ts;
  const bool vec_out = (a.Ha % 256) == 0, vec_in = (a.A % 8) == 0;
  if (a.k_out >= 0) {
    float sq = 0.f;
    for (int j = tid; j < a.Ha; j += nthr) {
      const float hv = __ldcg(hrow + static_cast<size_t>(j) * a.h_fs);
      hs[j] = hv * a.final_norm[j];
      sq += hv * hv;
    }
    sq = warp_sum(sq);
    if (lane == 0) sred[warp] = sq;
    sync();
    float tot = 0.f;
    for (int w = 0; w < nw; ++w) tot += sred[w];
    const float inv = rsqrtf(tot / a.Ha + a.eps);
    const float dt = -1.0f / a.steps;
    const float* sh = kMod ? final_shift : nullptr;
    for (int o = warp; o < a.A; o += nw) {
      const __nv_bfloat16* wr = a.W_out + static_cast<size_t>(o) * a.Ha;
      float acc = 0.f, accb = 0.f;   // accb: the modulated norm's shift through W_out
      if (vec_out) {   // lane reads 8 consecutive weights per 256-wide slice
        for (int j0 = lane * 8; j0 < a.Ha; j0 += 256) {
          const uint4 w8 = __ldg(reinterpret_cast<const uint4*>(wr + j0));
          const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&w8);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(w2[e]);
            acc += f.x * hs[j0 + 2 * e] + f.y * hs[j0 + 2 * e + 1];
            if (sh) accb += f.x * sh[j0 + 2 * e] + f.y * sh[j0 + 2 * e + 1];
          }
        }
      } else {
        for (int j = lane; j < a.Ha; j += 32) {
          acc += __bfloat162float(wr[j]) * hs[j];
          if (sh) accb += __bfloat162float(wr[j]) * sh[j];
        }
      }
      acc = warp_sum(acc);
      if (sh) accb = warp_sum(accb);
      if (lane == 0) {
        const float v = kMod ? acc * inv + (accb + a.b_out[o]) : acc * inv + a.b_out[o];
        float* xp = a.x + static_cast<size_t>(tok) * a.A + o;
        *xp = *xp + dt * v;
        if (a.vel) a.vel[(static_cast<size_t>(a.k_out) * a.tokens + tok) * a.A + o] = v;
      }
    }
    sync();
  }
  if (a.k_in >= 0) {
    if (tid < a.A) sx[tid] = a.x[static_cast<size_t>(tok) * a.A + tid];
    sync();
    const float t = 1.0f - static_cast<float>(a.k_in) / static_cast<float>(a.steps);
    const int half = a.Ha >> 1;
    const float kLog2_10000 = 13.287712379549449f;
    float sq = 0.f;
    for (int j = tid; j < a.Ha; j += nthr) {
      float e = a.b_in[j];
      const __nv_bfloat16* w = a.W_in + static_cast<size_t>(j) * a.A;
      if (vec_in) {
        for (int i0 = 0; i0 < a.A; i0 += 8) {
          const uint4 w8 = __ldg(reinterpret_cast<const uint4*>(w + i0));
          const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&w8);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(w2[q]);
            e += f.x * sx[i0 + 2 * q] + f.y * sx[i0 + 2 * q + 1];
          }
        }
      } else {
        for (int i = 0; i < a.A; ++i) e += __bfloat162float(w[i]) * sx[i];
      }
      if (!kMod) {
        const int fi = j < half ? j : j - half;
        const float arg = t * exp2f(-static_cast<float>(fi) / half * kLog2_10000);
        e += j < half ? sinf(arg) : cosf(arg);
      }
      hrow[static_cast<size_t>(j) * a.h_fs] = e;
      if (a.xn) a.xn[static_cast<size_t>(tok) * a.Ha + j] = __float2bfloat16_rn(a.attn_norm0[j] * e);
      sq += e * e;
    }
    if (a.ssq) {
      sq = warp_sum(sq);
      sync();
      if (lane == 0) sred[warp] = sq;
      sync();
      if (tid == 0) {
        float tot = 0.f;
        for (int w = 0; w < nw; ++w) tot += sred[w];
        a.ssq[tok] = tot;
      }
      for (int s = 1 + tid; s < a.n_slots; s += nthr) a.ssq[static_cast<size_t>(s) * a.tokens + tok] = 0.f;
    }
  }
}

// One CTA (256 threads) per action token; dynamic shared memory: Ha floats.  final_shift non-null
// selects the time-modulated step.
__global__ void __launch_bounds__(256) step_kernel(const StepArgs a, const float* final_shift) {
  __shared__ float sx[64];
  __shared__ float sred[8];
  extern __shared__ float step_hs[];
  pdl_launch_dependents();
  pdl_wait();
  if (final_shift)
    step_token<true>(a, blockIdx.x, threadIdx.x, 256, sx, sred, step_hs, [] { __syncthreads(); }, final_shift);
  else
    step_token<false>(a, blockIdx.x, threadIdx.x, 256, sx, sred, step_hs, [] { __syncthreads(); });
}

// ---------------------------------------------------------------- time modulation (DM0.5 page, section 5.2)
//
// The time-modulated action expert turns the flow time into a condition c(t) = W_to silu(W_ti tau(t) +
// b_ti) + b_to and every pre-norm into an adaptive RMSNorm whose scale, shift and gate are
// W_m silu(c) + b_m.  They depend only on t_k = 1 - k/K and the weights, so one pass per Euler loop
// builds them for all K steps (three GEMMs over K rows, below) instead of per step.

// row k of out: bf16 tau(t_k), t_k = 1 - k / steps, [sin(t w_i) | cos(t w_i)], w_i = 10000^(-i / (Ha/2))
__global__ void __launch_bounds__(256) tmod_tau_kernel(__nv_bfloat16* out, int steps, int Ha) {
  pdl_launch_dependents();
  pdl_wait();
  const int k = blockIdx.x, half = Ha >> 1;
  const float t = 1.0f - static_cast<float>(k) / static_cast<float>(steps);
  const float kLog2_10000 = 13.287712379549449f;
  for (int j = threadIdx.x; j < Ha; j += blockDim.x) {
    const int fi = j < half ? j : j - half;
    const float arg = t * exp2f(-static_cast<float>(fi) / half * kLog2_10000);
    out[static_cast<size_t>(k) * Ha + j] = __float2bfloat16_rn(j < half ? sinf(arg) : cosf(arg));
  }
}

// out[r][c] = bf16(silu(in[r][c] + bias[c])): the activation between the time MLP's layers, and the
// modulators' input silu(c)
__global__ void __launch_bounds__(256) tmod_bias_silu_kernel(const float* in, const float* bias, int cols,
                                                             __nv_bfloat16* out) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t r = blockIdx.x;
  for (int j = threadIdx.x; j < cols; j += blockDim.x) {
    const float v = in[r * cols + j] + bias[j];
    out[r * cols + j] = __float2bfloat16_rn(silu_f(v));
  }
}

// Finish the modulation table mod[k][0 .. L 6 Ha + 2 Ha) in place: add the bias, turn every scale g
// into 1 + g (the factor that multiplies x / rms(x)), and copy each layer's two shifts in bf16 to
// beta[l][0 attention | 1 MLP][k][Ha], the operands of the shift projections.  Per layer the rows are
// [attention: scale | shift | gate][MLP: scale | shift | gate]; the final norm's [scale | shift] close
// the row.
__global__ void __launch_bounds__(256) tmod_finish_kernel(float* mod, const float* bmod, int steps, int L, int Ha,
                                                          __nv_bfloat16* beta) {
  pdl_launch_dependents();
  pdl_wait();
  const int k = blockIdx.y;
  const int R = (6 * L + 2) * Ha;
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= R) return;
  float v = mod[static_cast<size_t>(k) * R + r] + bmod[r];
  const int l = r / (6 * Ha), q = r - l * 6 * Ha, part = q / Ha, j = q - part * Ha;
  if (part == 0 || part == 3) v += 1.f;   // scales (the final norm's scale is part 0 of "layer" L)
  if (l < L && (part == 1 || part == 4))
    beta[((static_cast<size_t>(l) * 2 + (part == 4)) * steps + k) * Ha + j] = __float2bfloat16_rn(v);
  mod[static_cast<size_t>(k) * R + r] = v;
}

// Failure-path self-test: one thread waits, with the library's bounded wait, on an mbarrier
// that nothing ever arrives on.  The wait gives up after `limit_ns`, the kernel records the
// timeout in the device error word and returns normally.
__global__ void wait_timeout_selftest_kernel(int* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait(&bar, 0, nullptr, limit_ns)) raise_error(err, kErrTimeoutProducer);
  }
}

// FP8 E4M3 row quantisation (the operands of the FP8 prefix-MLP GEMMs; DM0.5 page, section 6.3, with
// per-row scales).  Row r of x (bf16 or fp32), optionally times gain[c] and the row's pending RMSNorm
// factor 1/sqrt(sum of its ssq slots / cols + eps), is y[c]; scale[r] = amax(|y|) / 448 in fp32 (1 for an all-zero
// row) and q[r][c] = E4M3(y[c] / scale[r]), the quotient an IEEE fp32 division and the conversion
// round to nearest even, saturating.  One CTA of 256 threads per row, 16-byte loads (8 bf16 or 4
// fp32), cols a multiple of 8; the row is read twice, the second time from L1 / L2.  Used for the
// weights once (bf16 rows = output channels) and for the activations (fp32 rows = tokens).
template <typename T>
__device__ __forceinline__ void quant_load(const T* row, const float* gain, float rn, int v, float (&y)[16 / sizeof(T)]) {
  constexpr int kV = 16 / sizeof(T);
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(row) + v);
  if constexpr (sizeof(T) == 2) {
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(b[i]);
      y[2 * i] = f.x;
      y[2 * i + 1] = f.y;
    }
  } else {
    y[0] = __uint_as_float(u.x);
    y[1] = __uint_as_float(u.y);
    y[2] = __uint_as_float(u.z);
    y[3] = __uint_as_float(u.w);
  }
  if (gain) {
#pragma unroll
    for (int i = 0; i < kV; ++i) y[i] = y[i] * rn * __ldg(gain + v * kV + i);
  } else if (rn != 1.f) {
#pragma unroll
    for (int i = 0; i < kV; ++i) y[i] *= rn;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) quant_rows_e4m3_kernel(const T* x, int rows, int cols, const float* gain,
                                                              const float* ssq, int ssq_slots, int ssq_stride,
                                                              float inv_cols, float eps, uint8_t* q, float* scale) {
  constexpr int kV = 16 / sizeof(T);
  __shared__ float red[8];
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x;
  if (row >= rows) return;
  const T* src = x + static_cast<size_t>(row) * cols;
  float rn = 1.f;
  if (ssq) {   // partial sums of squares of the row, added in slot order
    float ss = 0.f;
    for (int q2 = 0; q2 < ssq_slots; ++q2) ss += __ldcg(ssq + static_cast<size_t>(q2) * ssq_stride + row);
    rn = rsqrtf(ss * inv_cols + eps);
  }
  const int nvec = cols / kV;
  float amax = 0.f;
  for (int v = threadIdx.x; v < nvec; v += 256) {
    float y[kV];
    quant_load(src, gain, rn, v, y);
#pragma unroll
    for (int i = 0; i < kV; ++i) amax = fmaxf(amax, fabsf(y[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float s = amax > 0.f ? amax / 448.f : 1.f;
  if (threadIdx.x == 0) scale[row] = s;
  uint8_t* dst = q + static_cast<size_t>(row) * cols;
  for (int v = threadIdx.x; v < nvec; v += 256) {
    float y[kV];
    quant_load(src, gain, rn, v, y);
    uint32_t w[kV / 4];
#pragma unroll
    for (int i = 0; i < kV / 4; ++i) {
      w[i] = 0u;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w[i] |= static_cast<uint32_t>(__nv_cvt_float_to_fp8(y[4 * i + j] / s, __NV_SATFINITE, __NV_E4M3)) << (8 * j);
    }
    if constexpr (kV == 8)
      reinterpret_cast<uint2*>(dst)[v] = make_uint2(w[0], w[1]);
    else
      reinterpret_cast<uint32_t*>(dst)[v] = w[0];
  }
}

// (cos, sin) of every (position, frequency): position-major in `tab` [max_pos][half] and the same
// values dimension-major in `tab_t` [half][max_pos], where the 32 consecutive tokens of a warp read
// one frequency as two 128-byte lines
__global__ void rope_table_kernel(float2* tab, float2* tab_t, int max_pos, int half, double log_theta) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= max_pos * half) return;
  const int pos = idx / half, i = idx - (idx / half) * half;
  const double inv_freq = exp(-(2.0 * i / (2.0 * half)) * log_theta);
  const double ang = static_cast<double>(pos) * inv_freq;
  const float2 cs = make_float2(static_cast<float>(cos(ang)), static_cast<float>(sin(ang)));
  tab[idx] = cs;
  tab_t[static_cast<size_t>(i) * max_pos + pos] = cs;
}

}  // namespace dm0
