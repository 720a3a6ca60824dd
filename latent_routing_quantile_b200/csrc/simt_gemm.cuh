// fp32 FFMA GEMM for the fp32 layer configuration: C = A B^T with both operands K-contiguous.
// Tensor-core tf32 keeps 10 mantissa bits, which cannot meet fp32 accuracy, so the fp32 layer
// runs its products here.  Tile 128 x 32 x 32, 256 threads, 4 x 4 outputs per thread.
// Same A/B conventions and grouped-tile table (padded expert layout) as the tensor-core engine;
// an optional second B operand (dual mode) gives the gate and linear halves of a SwiGLU in one
// pass.
#pragma once

#include "common.cuh"

namespace lmoe {

enum SimtEpilogue : int {
  SE_STORE = 0,   // out = acc * (row_scale ? row_scale[row] : 1)
  SE_SWIGLU = 1,  // dual: out = silu(rs * acc0) * (rs * acc1)
  SE_ROUTER = 2,  // out = sigmoid(acc + col_bias[col])
};

struct SimtParams {
  const float* A0;
  int lda0, K0;  // columns [0, K0) of A
  const float* A1;
  int lda1, K1;  // columns [K0, K0 + K1) of A
  int a_rows;    // rows of A that exist (loads past it read zero)
  const float* B0;
  const float* B1;
  int ldb;
  long long b_group_stride;  // grouped: elements between experts' B matrices
  int M, N;
  int grouped;
  const int2* mtile_table;
  const int* num_mtiles;
  float* out;
  int ldo;
  const float* row_scale;
  const float* col_bias;
  uint32_t* status;
};

template <int EPI>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtParams p) {
  constexpr int BM = 128, BN = 32, BK = 32;
  constexpr bool kDual = (EPI == SE_SWIGLU);
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  __shared__ float Bs1[kDual ? BK : 1][BN + 4];

  pdl_wait();
  pdl_trigger();
  int row0, row_end, e = 0;
  if (p.grouped) {
    if ((int)blockIdx.y >= *p.num_mtiles) return;
    int2 er = p.mtile_table[blockIdx.y];
    e = er.x & 0xFFFF;  // the high half holds the tile's valid rows
    row0 = er.y;
    row_end = row0 + BM;  // padded expert layout: the whole tile belongs to expert e
  } else {
    row0 = blockIdx.y * BM;
    row_end = p.M;
  }
  const int n0 = blockIdx.x * BN;
  const float* B0 = p.B0 + (long long)e * p.b_group_stride;
  const float* B1 = kDual ? p.B1 + (long long)e * p.b_group_stride : nullptr;
  const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
  float acc[4][4] = {}, acc1[4][4] = {};
  const int K = p.K0 + p.K1;

  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int i = 0; i < (BM * BK) / 256; ++i) {
      int idx = tid + i * 256, r = idx / BK, kk = idx % BK, row = row0 + r, k = k0 + kk;
      float v = 0.f;
      if (row < p.a_rows) v = (k < p.K0) ? p.A0[(long long)row * p.lda0 + k]
                                         : p.A1[(long long)row * p.lda1 + (k - p.K0)];
      As[kk][r] = v;
    }
#pragma unroll
    for (int i = 0; i < (BN * BK) / 256; ++i) {
      int idx = tid + i * 256, n = idx / BK, kk = idx % BK;
      Bs[kk][n] = B0[(long long)(n0 + n) * p.ldb + k0 + kk];
      if constexpr (kDual) Bs1[kk][n] = B1[(long long)(n0 + n) * p.ldb + k0 + kk];
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b[j] = Bs[kk][tx * 4 + j];
        if constexpr (kDual) b1[j] = Bs1[kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
          if constexpr (kDual) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }

  bool nan = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = row0 + ty * 4 + i;
    if (row >= row_end) continue;
    const float rs = p.row_scale ? p.row_scale[row] : 1.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + tx * 4 + j;
      float v;
      if constexpr (EPI == SE_STORE) {
        v = acc[i][j] * rs;
      } else if constexpr (EPI == SE_SWIGLU) {
        v = siluf(acc[i][j] * rs) * (acc1[i][j] * rs);
      } else {
        v = sigmoidf_acc(acc[i][j] + p.col_bias[col]);
        nan |= (v != v);
      }
      p.out[(long long)row * p.ldo + col] = v;
    }
  }
  if (nan) set_status(p.status, LMOE_STATUS_NAN_SCORE);
}

}  // namespace lmoe
