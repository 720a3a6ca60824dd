// Memory-bound kernels of the layer backward (the gradient of sum(y * dy) for the layer's
// forward; its GEMMs run on the tensor-core engine in tc_gemm.cuh).  Notation per token t:
//   r = (mean_j x_j^2 + eps)^(-1/2), x_hat = gain * x * r, h = x_hat W_down^T,
//   s = sigmoid(h W_r^T + c), g_i = s_{e_i} / S with S = sum_i s_{e_i},
//   o_i = SwiGLU_{e_i}(h), z = sum_i g_i o_i, y = z W_up^T + SwiGLU_shared(x_hat).
// No gradient flows through the expert choice or into the balancing bias b: the choice is
// piecewise constant in every input, and b only reroutes ("Pretraining a Mini Kimi K3",
// capsule 16; "KimiK3MoE 架构轻量化复刻演示上线", Tab 8-10: the gates are the renormalised
// unbiased scores).
#pragma once

#include "common.cuh"

namespace lmoe {

// x_hat = bf16(gain * x * r), the operand of the W_down and shared-expert weight gradients.
__global__ void __launch_bounds__(256) xhat_kernel(const bf16* __restrict__ x, const bf16* __restrict__ gain,
                                                   const float* __restrict__ r, long long T, int d,
                                                   bf16* __restrict__ xh) {
  pdl_wait();
  pdl_trigger();
  const long long nv = T * d / 8;
  for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < nv; v += (long long)gridDim.x * blockDim.x) {
    const long long t = v * 8 / d;
    const int c = (int)(v * 8 - t * d);
    const uint4 q = reinterpret_cast<const uint4*>(x)[v];
    uint4 gq = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);  // 1.0 pairs
    if (gain) gq = reinterpret_cast<const uint4*>(gain)[c / 8];
    const float rt = r[t];
    const bf16* xe = reinterpret_cast<const bf16*>(&q);
    const bf16* ge = reinterpret_cast<const bf16*>(&gq);
    uint4 out;
    uint32_t* ow = &out.x;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      ow[j] = pack_bf16x2(bf2f(xe[2 * j]) * bf2f(ge[2 * j]) * rt, bf2f(xe[2 * j + 1]) * bf2f(ge[2 * j + 1]) * rt);
    reinterpret_cast<uint4*>(xh)[v] = out;
  }
}

// Combine and gate backward, one warp per token.  With dz = dL/dz:
//   dL/dg_i = dz . o_i;   dL/do_i = g_i dz   (written to the pair's row of the padded layout);
//   dL/ds_i = (dL/dg_i - sum_j g_j dL/dg_j) / S  (g_i = s_i / S; unchosen scores get nothing);
//   dL/dlogit_i = dL/ds_i s_i (1 - s_i)  (s = sigmoid of the logit).
// dlogit [T, E] bf16 is written whole (zeros but for the k chosen experts) for the router's
// GEMMs; dlp holds each pair's logit gradient in fp32 at its padded row, for the column offsets'
// gradient.
__global__ void __launch_bounds__(256) combine_bwd_kernel(const bf16* __restrict__ dz, const bf16* __restrict__ o,
                                                          const int* __restrict__ prow,
                                                          const float* __restrict__ gates,
                                                          const int* __restrict__ idx, const float* __restrict__ s,
                                                          int ntok, int k, int l, int E, bf16* __restrict__ d_o,
                                                          bf16* __restrict__ dlogit, float* __restrict__ dlp) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= ntok) return;
  const int r_l = lane < k ? prow[(size_t)t * k + lane] : 0;
  const float g_l = lane < k ? gates[(size_t)t * k + lane] : 0.f;
  const int e_l = lane < k ? idx[(size_t)t * k + lane] : 0;
  const float s_l = lane < k ? s[(size_t)t * E + e_l] : 0.f;
  const int nvec = l / 8;
  const uint4* dzr = reinterpret_cast<const uint4*>(dz + (size_t)t * l);
  float dg_l = 0.f;
  for (int i = 0; i < k; ++i) {
    const int row = __shfl_sync(kFull, r_l, i);
    const float gi = __shfl_sync(kFull, g_l, i);
    const uint4* orow = reinterpret_cast<const uint4*>(o + (size_t)row * l);
    uint4* drow = reinterpret_cast<uint4*>(d_o + (size_t)row * l);
    float acc = 0.f;
    for (int v = lane; v < nvec; v += 32) {
      const uint4 zq = dzr[v], oq = orow[v];
      const bf16* ze = reinterpret_cast<const bf16*>(&zq);
      const bf16* oe = reinterpret_cast<const bf16*>(&oq);
      uint4 out;
      uint32_t* ow = &out.x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float z0 = bf2f(ze[2 * j]), z1 = bf2f(ze[2 * j + 1]);
        acc = fmaf(z0, bf2f(oe[2 * j]), acc);
        acc = fmaf(z1, bf2f(oe[2 * j + 1]), acc);
        ow[j] = pack_bf16x2(gi * z0, gi * z1);
      }
      drow[v] = out;
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(kFull, acc, off);
    if (lane == i) dg_l = acc;
  }
  float S = s_l, G = g_l * dg_l;
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    S += __shfl_xor_sync(kFull, S, off);
    G += __shfl_xor_sync(kFull, G, off);
  }
  const float ds = (dg_l - G) / S;
  const float dl = ds * s_l * (1.f - s_l);
  uint4* lrow = reinterpret_cast<uint4*>(dlogit + (size_t)t * E);
  for (int v = lane; v < E / 8; v += 32) lrow[v] = make_uint4(0, 0, 0, 0);
  __syncwarp();
  if (lane < k) {
    dlogit[(size_t)t * E + e_l] = __float2bfloat16_rn(dl);
    dlp[r_l] = dl;
  }
}

// Zeroes the rows [n_e, n_e rounded up to 64) of each expert's block of the padded layout in up to
// three matrices (columns c0, c1, c2; a null matrix is skipped), so that products whose K runs
// over an expert's rows in whole 64-row blocks add nothing from rows past its last pair.
__global__ void __launch_bounds__(256) pad_zero_kernel(const int* __restrict__ offsets, const int* __restrict__ pad_delta,
                                                       const int* __restrict__ counts, bf16* __restrict__ m0, int c0,
                                                       bf16* __restrict__ m1, int c1, bf16* __restrict__ m2, int c2) {
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x;
  const int n = counts[e];
  const long long first = (long long)offsets[e] + pad_delta[e] + n;
  const int rows = ((n + 63) & ~63) - n;
  bf16* mats[3] = {m0, m1, m2};
  const int cols[3] = {c0, c1, c2};
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    if (!mats[m]) continue;
    const int nv = cols[m] / 8;
    uint4* base = reinterpret_cast<uint4*>(mats[m] + first * cols[m]);
    for (int i = threadIdx.x; i < rows * nv; i += blockDim.x) base[i] = make_uint4(0, 0, 0, 0);
  }
}

// dL/dc_e = sum of the logit gradients of expert e's pairs (its rows of the padded layout), one
// warp per expert.
__global__ void __launch_bounds__(256) bias_grad_kernel(const int* __restrict__ offsets, const int* __restrict__ pad_delta,
                                                        const int* __restrict__ counts, const float* __restrict__ dlp,
                                                        int E, float* __restrict__ dc) {
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (e >= E) return;
  const long long first = (long long)offsets[e] + pad_delta[e];
  const int n = counts[e];
  float acc = 0.f;
  for (int i = lane; i < n; i += 32) acc += dlp[first + i];
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(kFull, acc, off);
  if (lane == 0) dc[e] = acc;
}

// dh[t] = dh_router[t] + sum_i dh_expert[row of pair (t, i)], one warp per token; fp32 sums, the
// result rounded to bf16 (the operand of the W_down gradient and of dL/dx_hat).
__global__ void __launch_bounds__(256) scatter_dh_kernel(const float* __restrict__ dhr, const bf16* __restrict__ dhe,
                                                         const int* __restrict__ prow, int ntok, int k, int l,
                                                         bf16* __restrict__ dh) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= ntok) return;
  const int r_l = lane < k ? prow[(size_t)t * k + lane] : 0;
  const int nvec = l / 8;
  for (int v0 = 0; v0 < nvec; v0 += 32) {
    const int v = v0 + lane;
    const bool act = v < nvec;
    float acc[8];
    if (act) {
      const float4 a = reinterpret_cast<const float4*>(dhr + (size_t)t * l)[2 * v];
      const float4 b = reinterpret_cast<const float4*>(dhr + (size_t)t * l)[2 * v + 1];
      acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
      acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
    }
    for (int i = 0; i < k; ++i) {
      const int row = __shfl_sync(kFull, r_l, i);
      if (!act) continue;
      const uint4 q = reinterpret_cast<const uint4*>(dhe + (size_t)row * l)[v];
      const bf16* e = reinterpret_cast<const bf16*>(&q);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += bf2f(e[j]);
    }
    if (!act) continue;
    uint4 out;
    uint32_t* ow = &out.x;
#pragma unroll
    for (int j = 0; j < 4; ++j) ow[j] = pack_bf16x2(acc[2 * j], acc[2 * j + 1]);
    reinterpret_cast<uint4*>(dh + (size_t)t * l)[v] = out;
  }
}

// RMSNorm backward over a block of kRmsRows tokens.  With gdx = gain * dL/dx_hat:
//   dL/dx = gdx r - x r^3 / d * sum_m gdx_m x_m;   dL/dgain_m = sum_t dL/dx_hat_m x_m r.
// Phase 1 (a warp per token) forms each row's sum; phase 2 (threads over columns, tokens in
// order) writes dL/dx and this block's partial dL/dgain, so the sums need no atomics.
constexpr int kRmsRows = 64;
__global__ void __launch_bounds__(256) rms_bwd_kernel(const bf16* __restrict__ x, const bf16* __restrict__ gain,
                                                      const float* __restrict__ r, const float* __restrict__ dxh,
                                                      int ntok, int d, float* __restrict__ dx,
                                                      float* __restrict__ gpart) {
  pdl_wait();
  pdl_trigger();
  __shared__ float dot[kRmsRows];
  const int t0 = blockIdx.x * kRmsRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int tt = warp; tt < kRmsRows; tt += 8) {
    const int t = t0 + tt;
    float acc = 0.f;
    if (t < ntok)
      for (int c = lane; c < d; c += 32) {
        const float gm = gain ? bf2f(gain[c]) : 1.f;
        acc = fmaf(gm * dxh[(size_t)t * d + c], bf2f(x[(size_t)t * d + c]), acc);
      }
#pragma unroll
    for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(kFull, acc, off);
    if (lane == 0) dot[tt] = acc;
  }
  __syncthreads();
  const float inv_d = 1.f / (float)d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float gm = gain ? bf2f(gain[c]) : 1.f;
    float ga = 0.f;
    for (int tt = 0; tt < kRmsRows; ++tt) {
      const int t = t0 + tt;
      if (t >= ntok) break;
      const float rt = r[t];
      const float xv = bf2f(x[(size_t)t * d + c]);
      const float g = dxh[(size_t)t * d + c];
      dx[(size_t)t * d + c] = gm * g * rt - xv * rt * rt * rt * inv_d * dot[tt];
      ga = fmaf(g * xv, rt, ga);
    }
    gpart[(size_t)blockIdx.x * d + c] = ga;
  }
}

// dL/dgain = the sum of the blocks' partial sums, in block order.
__global__ void __launch_bounds__(256) colsum_kernel(const float* __restrict__ part, int nrows, int d,
                                                     float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= d) return;
  float acc = 0.f;
  for (int i = 0; i < nrows; ++i) acc += part[(size_t)i * d + c];
  out[c] = acc;
}

}  // namespace lmoe
