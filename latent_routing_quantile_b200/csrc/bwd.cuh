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
// Phase 1 (a warp per token, 16-byte loads) forms each row's sum; phase 2 (a thread per 8
// columns, the block's tokens in order) writes dL/dx and this block's partial dL/dgain, so the
// sums need no atomics and come out the same every run.
constexpr int kRmsRows = 32;
__device__ __forceinline__ void load8_f32(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8_bf16(const bf16* p, float (&v)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const bf16* e = reinterpret_cast<const bf16*>(&q);
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = bf2f(e[j]);
}
__global__ void __launch_bounds__(256) rms_bwd_kernel(const bf16* __restrict__ x, const bf16* __restrict__ gain,
                                                      const float* __restrict__ r, const float* __restrict__ dxh,
                                                      int ntok, int d, float* __restrict__ dx,
                                                      float* __restrict__ gpart) {
  pdl_wait();
  pdl_trigger();
  __shared__ float dot[kRmsRows];
  const int t0 = blockIdx.x * kRmsRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = d / 8;
  for (int tt = warp; tt < kRmsRows; tt += 8) {
    const int t = t0 + tt;
    float acc = 0.f;
    if (t < ntok)
      for (int v = lane; v < nv; v += 32) {
        float xv[8], gv[8], gm[8];
        load8_bf16(x + (size_t)t * d + 8 * v, xv);
        load8_f32(dxh + (size_t)t * d + 8 * v, gv);
        if (gain) load8_bf16(gain + 8 * v, gm);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc = fmaf((gain ? gm[j] : 1.f) * gv[j], xv[j], acc);
      }
#pragma unroll
    for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(kFull, acc, off);
    if (lane == 0) dot[tt] = acc;
  }
  __syncthreads();
  const float inv_d = 1.f / (float)d;
  const int nt = min(kRmsRows, ntok - t0);
  for (int v = threadIdx.x; v < nv; v += blockDim.x) {
    float gm[8], ga[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) ga[j] = 0.f;
    if (gain) load8_bf16(gain + 8 * v, gm);
    else
#pragma unroll
      for (int j = 0; j < 8; ++j) gm[j] = 1.f;
#pragma unroll 4
    for (int tt = 0; tt < nt; ++tt) {
      const int t = t0 + tt;
      const float rt = r[t];
      const float cr = rt * rt * rt * inv_d * dot[tt];
      float xv[8], gv[8];
      load8_bf16(x + (size_t)t * d + 8 * v, xv);
      load8_f32(dxh + (size_t)t * d + 8 * v, gv);
      float o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        o[j] = gm[j] * gv[j] * rt - xv[j] * cr;
        ga[j] = fmaf(gv[j] * xv[j], rt, ga[j]);
      }
      float4* dst = reinterpret_cast<float4*>(dx + (size_t)t * d + 8 * v);
      dst[0] = make_float4(o[0], o[1], o[2], o[3]);
      dst[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
    float4* gp = reinterpret_cast<float4*>(gpart + (size_t)blockIdx.x * d + 8 * v);
    gp[0] = make_float4(ga[0], ga[1], ga[2], ga[3]);
    gp[1] = make_float4(ga[4], ga[5], ga[6], ga[7]);
  }
}

// dL/dgain = the sum of the blocks' partial sums: a block per 32 columns, its 8 warps summing
// interleaved rows, then the 8 sums added in a fixed order.
__global__ void __launch_bounds__(256) colsum_kernel(const float* __restrict__ part, int nrows, int d,
                                                     float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sm[8][33];
  const int c = blockIdx.x * 32 + (threadIdx.x & 31), y = threadIdx.x >> 5;
  float acc = 0.f;
  if (c < d) {
#pragma unroll 8
    for (int i = y; i < nrows; i += 8) acc += part[(size_t)i * d + c];
  }
  sm[y][threadIdx.x & 31] = acc;
  __syncthreads();
  if (y == 0 && c < d) {
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) s += sm[j][threadIdx.x];
    out[c] = s;
  }
}

}  // namespace lmoe
