// Small bandwidth-trivial kernels around the GEMM/attention chain:
//   rows_prep    : residual stream in (bf16 prefix embeddings or fp32), first
//                  pending RMSNorm operand bf16(g * h) and its sum of squares.
//   step_kernel  : per action token, the flow-matching step boundary
//                  (DM0.5 page, sections 5.2-5.3): velocity
//                  v = RMSNorm_final(h) W_out^T + b_out, Euler update
//                  x <- x + dt v with dt = -1/K, then the next step's input
//                  e = x W_in^T + b_in + tau(t) with t = 1 - k/K.
//   rope_table   : (cos, sin) of position * theta^(-2i/D), in double precision.
#pragma once
#include "ptx.cuh"

namespace dm0 {

// h[row] = in[row]; xn[row] = bf16(gain * h); ssq[0][row] = sum h^2; ssq[s][row] = 0 for s >= 1.
// One warp per row.
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
  float* h;                    // [tokens][Ha] action residual stream
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

// One CTA (256 threads) per action token.
__global__ void __launch_bounds__(256) step_kernel(const StepArgs a) {
  __shared__ float sx[64];
  __shared__ float sred[8];
  pdl_launch_dependents();
  pdl_wait();
  const int tok = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* hrow = a.h + static_cast<size_t>(tok) * a.Ha;
  if (a.k_out >= 0) {
    float sq = 0.f;
    for (int j = tid; j < a.Ha; j += 256) sq += hrow[j] * hrow[j];
    sq = warp_sum(sq);
    if (lane == 0) sred[warp] = sq;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += sred[w];
    const float inv = rsqrtf(tot / a.Ha + a.eps);
    const float dt = -1.0f / a.steps;
    for (int o = warp; o < a.A; o += 8) {
      float acc = 0.f;
      for (int j = lane; j < a.Ha; j += 32)
        acc += __bfloat162float(a.W_out[static_cast<size_t>(o) * a.Ha + j]) * (hrow[j] * a.final_norm[j]);
      acc = warp_sum(acc);
      if (lane == 0) {
        const float v = acc * inv + a.b_out[o];
        float* xp = a.x + static_cast<size_t>(tok) * a.A + o;
        *xp = *xp + dt * v;
        if (a.vel) a.vel[(static_cast<size_t>(a.k_out) * a.tokens + tok) * a.A + o] = v;
      }
    }
    __syncthreads();
  }
  if (a.k_in >= 0) {
    if (tid < a.A) sx[tid] = a.x[static_cast<size_t>(tok) * a.A + tid];
    __syncthreads();
    const float t = 1.0f - static_cast<float>(a.k_in) / static_cast<float>(a.steps);
    const int half = a.Ha >> 1;
    const float kLog2_10000 = 13.287712379549449f;
    float sq = 0.f;
    for (int j = tid; j < a.Ha; j += 256) {
      float e = a.b_in[j];
      const __nv_bfloat16* w = a.W_in + static_cast<size_t>(j) * a.A;
      for (int i = 0; i < a.A; ++i) e += __bfloat162float(w[i]) * sx[i];
      const int fi = j < half ? j : j - half;
      const float arg = t * exp2f(-static_cast<float>(fi) / half * kLog2_10000);
      e += j < half ? sinf(arg) : cosf(arg);
      hrow[j] = e;
      a.xn[static_cast<size_t>(tok) * a.Ha + j] = __float2bfloat16_rn(a.attn_norm0[j] * e);
      sq += e * e;
    }
    sq = warp_sum(sq);
    __syncthreads();
    if (lane == 0) sred[warp] = sq;
    __syncthreads();
    if (tid == 0) {
      float tot = 0.f;
      for (int w = 0; w < 8; ++w) tot += sred[w];
      a.ssq[tok] = tot;
    }
    for (int s = 1 + tid; s < a.n_slots; s += 256) a.ssq[static_cast<size_t>(s) * a.tokens + tok] = 0.f;
  }
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

__global__ void rope_table_kernel(float2* tab, int max_pos, int half, double log_theta) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= max_pos * half) return;
  const int pos = idx / half, i = idx - (idx / half) * half;
  const double inv_freq = exp(-(2.0 * i / (2.0 * half)) * log_theta);
  const double ang = static_cast<double>(pos) * inv_freq;
  tab[idx] = make_float2(static_cast<float>(cos(ang)), static_cast<float>(sin(ang)));
}

}  // namespace dm0
