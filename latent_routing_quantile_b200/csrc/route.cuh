// Memory-bound kernels of the layer: RMSNorm reciprocal, biased top-k with gates and stable
// per-block ranks, the dispatch plan (offsets, per-block bases, grouped-GEMM tile table), the
// permutation gather, the QB score histogram, the weighted combine, and the QB update.
#pragma once

#include <climits>

#include "common.cuh"

namespace lmoe {

constexpr int kTokBlock = 128;     // tokens per routing block: a rank bitmask is 4 words
constexpr int kTileRows = 128;     // rows per grouped-GEMM M-tile
constexpr unsigned kFull = 0xffffffffu;

// --------------------------------------------------------------------------- RMSNorm
// r_t = 1 / sqrt(mean_j x_tj^2 + eps); one warp per token, squares summed in fp64.
template <typename T>
__global__ void __launch_bounds__(256) rms_kernel(const T* __restrict__ x, int ntok, int d, float eps,
                                                  float* __restrict__ r) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= ntok) return;
  constexpr int VEC = 16 / sizeof(T);
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)row * d);
  double acc = 0.0;
  for (int v = lane; v < d / VEC; v += 32) {
    uint4 q = xr[v];
    const T* e = reinterpret_cast<const T*>(&q);
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      double f = (double)to_f<T>(e[j]);
      acc += f * f;
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(kFull, acc, off);
  if (lane == 0) r[row] = (float)(1.0 / sqrt(acc / d + (double)eps));
}

// --------------------------------------------------------------------------- top-k
// One warp per token, 16 tokens per warp, kTokBlock tokens per block.  k rounds of a warp
// arg-max of u = s + b over the experts not yet taken; order: larger u, then lower index.
// Gates are the chosen unbiased s divided by their sum.  Each choice sets the token's bit in
// the expert's shared bitmask; a token's rank inside the block for expert e is the number of
// set bits below its own, which gives a stable (token-ascending) order without atomics on the
// order.  Per-block counts go to blkcnt and are summed into counts.
template <int NJ>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ s, const float* __restrict__ bias,
                                                   int ntok, int E, int k, int* __restrict__ idx,
                                                   float* __restrict__ gates, int* __restrict__ rank,
                                                   int* __restrict__ blkcnt, int* __restrict__ counts,
                                                   uint32_t* status) {
  extern __shared__ uint32_t mask[];  // [E][4]
  const int blk = blockIdx.x, t0 = blk * kTokBlock;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < E * 4; i += blockDim.x) mask[i] = 0;
  float bj[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = j * 32 + lane;
    bj[j] = e < E ? bias[e] : 0.f;
  }
  __syncthreads();

  bool nan = false;
  for (int q = 0; q < kTokBlock / 8; ++q) {
    const int t = t0 + warp * (kTokBlock / 8) + q;
    if (t >= ntok) break;
    float u[NJ], sv[NJ];
    uint32_t taken = 0;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = j * 32 + lane;
      if (e < E) {
        const float v = s[(size_t)t * E + e];
        if (v != v) {
          nan = true;
          u[j] = -INFINITY;
          sv[j] = 0.f;
        } else {
          u[j] = v + bj[j];
          sv[j] = v;
        }
      } else {
        u[j] = -INFINITY;
        sv[j] = 0.f;
        taken |= 1u << j;
      }
    }
    int my_sel = -1;
    float my_s = 0.f;
    for (int i = 0; i < k; ++i) {
      float bu = 0.f, bs = 0.f;
      int be = INT_MAX;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        if (!((taken >> j) & 1u) && (be == INT_MAX || u[j] > bu)) {
          bu = u[j];
          be = j * 32 + lane;
          bs = sv[j];
        }
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        const float ou = __shfl_xor_sync(kFull, bu, off);
        const int oe = __shfl_xor_sync(kFull, be, off);
        const float os = __shfl_xor_sync(kFull, bs, off);
        if (oe != INT_MAX && (be == INT_MAX || ou > bu || (ou == bu && oe < be))) {
          bu = ou;
          be = oe;
          bs = os;
        }
      }
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      if (lane == i) {
        my_sel = be;
        my_s = bs;
      }
    }
    float ssum = lane < k ? my_s : 0.f;
#pragma unroll
    for (int off = 16; off; off >>= 1) ssum += __shfl_xor_sync(kFull, ssum, off);
    if (lane < k) {
      idx[(size_t)t * k + lane] = my_sel;
      gates[(size_t)t * k + lane] = my_s / ssum;
      const int tl = t - t0;
      atomicOr(&mask[my_sel * 4 + (tl >> 5)], 1u << (tl & 31));
    }
  }
  if (nan) set_status(status, LMOE_STATUS_NAN_SCORE);
  __syncthreads();

  for (int q = 0; q < kTokBlock / 8; ++q) {
    const int t = t0 + warp * (kTokBlock / 8) + q;
    if (t >= ntok) break;
    if (lane < k) {
      const int e = idx[(size_t)t * k + lane];
      const int tl = t - t0, w = tl >> 5;
      int r = __popc(mask[e * 4 + w] & ((1u << (tl & 31)) - 1u));
      for (int ww = 0; ww < w; ++ww) r += __popc(mask[e * 4 + ww]);
      rank[(size_t)t * k + lane] = r;
    }
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = __popc(mask[e * 4]) + __popc(mask[e * 4 + 1]) + __popc(mask[e * 4 + 2]) +
                  __popc(mask[e * 4 + 3]);
    blkcnt[(size_t)blk * E + e] = c;
    if (c) atomicAdd(&counts[e], c);
  }
}

// --------------------------------------------------------------------------- dispatch plan
// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_exclusive_scan_1024(int v, int* sh /*[32]*/, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(kFull, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = sh[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFull, w, off);
      if (lane >= off) w += y;
    }
    sh[lane] = w;
  }
  __syncthreads();
  const int incl = x + (warp > 0 ? sh[warp - 1] : 0);
  *total = sh[31];
  __syncthreads();
  return incl - v;
}

// Grid: ceil(E/32) blocks of 1024 threads.  Every block recomputes the expert offsets (the
// exclusive scan of counts); block 0 stores them and the grouped-GEMM tile table; each block
// then fills blkbase[b][e] = off[e] + sum_{b' < b} blkcnt[b'][e] for its 32 experts.
__global__ void __launch_bounds__(1024) plan_kernel(const int* __restrict__ counts,
                                                    const int* __restrict__ blkcnt, int nblk, int E,
                                                    int* __restrict__ offsets, int* __restrict__ blkbase,
                                                    int2* __restrict__ mtiles, int* __restrict__ num_mtiles) {
  __shared__ int sh[32];
  __shared__ int s_off[1024];
  __shared__ int part[32][33];
  const int tid = threadIdx.x;
  const int c = tid < E ? counts[tid] : 0;
  int total;
  const int off = block_exclusive_scan_1024(c, sh, &total);
  s_off[tid] = off;
  if (blockIdx.x == 0) {
    if (tid < E) offsets[tid] = off;
    if (tid == 0) offsets[E] = total;
    const int mt = (c + kTileRows - 1) / kTileRows;
    int mt_total;
    const int mt_start = block_exclusive_scan_1024(mt, sh, &mt_total);
    for (int j = 0; j < mt; ++j) mtiles[mt_start + j] = make_int2(tid, off + j * kTileRows);
    if (tid == 0) *num_mtiles = mt_total;
  }
  __syncthreads();
  const int tx = tid & 31, ty = tid >> 5;
  const int e = blockIdx.x * 32 + tx;
  const int chunk = (nblk + 31) / 32;
  const int b0 = ty * chunk, b1 = min(nblk, b0 + chunk);
  int sum = 0;
  if (e < E)
    for (int b = b0; b < b1; ++b) sum += blkcnt[(size_t)b * E + e];
  part[ty][tx] = sum;
  __syncthreads();
  if (e < E) {
    int run = s_off[e];
    for (int q = 0; q < ty; ++q) run += part[q][tx];
    for (int b = b0; b < b1; ++b) {
      const int v = blkcnt[(size_t)b * E + e];
      blkbase[(size_t)b * E + e] = run;
      run += v;
    }
  }
}

// --------------------------------------------------------------------------- gather
// One warp per (token, slot): its permuted row pos = blkbase[block][e] + rank; records
// perm[pos] = token and inv[(t, i)] = pos, and copies the token's latent row into A_perm[pos].
template <typename T>
__global__ void __launch_bounds__(256) gather_kernel(const T* __restrict__ src, int ld_src, int l,
                                                     const int* __restrict__ idx, const int* __restrict__ rank,
                                                     const int* __restrict__ blkbase, int ntok, int E, int k,
                                                     int* __restrict__ perm, int* __restrict__ inv,
                                                     T* __restrict__ dst, uint32_t* status) {
  const int pair = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (pair >= ntok * k) return;
  const int t = pair / k, e = idx[pair];
  if (e < 0 || e >= E) {
    if (lane == 0) set_status(status, LMOE_STATUS_BAD_INDEX);
    return;
  }
  const int pos = blkbase[(size_t)(t / kTokBlock) * E + e] + rank[pair];
  if (pos < 0 || pos >= ntok * k) {
    if (lane == 0) set_status(status, LMOE_STATUS_BAD_INDEX);
    return;
  }
  if (lane == 0) {
    inv[pair] = pos;
    perm[pos] = t;
  }
  constexpr int VEC = 16 / sizeof(T);
  const uint4* s4 = reinterpret_cast<const uint4*>(src + (size_t)t * ld_src);
  uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)pos * l);
  for (int v = lane; v < l / VEC; v += 32) d4[v] = s4[v];
}

// --------------------------------------------------------------------------- QB histogram
// Each block owns G experts' 4096 bins in shared memory, reads their columns of s over all
// tokens, then adds its bins into the global histogram (no other block touches those rows).
// bin = min(floor(s * 4096), 4095); a NaN score counts in bin 0 (and was flagged by top-k).
__global__ void __launch_bounds__(1024) hist_kernel(const float* __restrict__ s, int ntok, int E, int G,
                                                    uint32_t* __restrict__ hist, long long* ntok_acc) {
  extern __shared__ uint32_t sh[];  // [G][4096]
  const int e0 = blockIdx.x * G, g_count = min(G, E - e0);
  for (int i = threadIdx.x; i < g_count * LMOE_NBINS; i += blockDim.x) sh[i] = 0;
  __syncthreads();
  const long long n = (long long)ntok * g_count;
  for (long long p = threadIdx.x; p < n; p += blockDim.x) {
    const int t = (int)(p / g_count), g = (int)(p - (long long)t * g_count);
    const float v = s[(size_t)t * E + e0 + g];
    const int bin = v >= 0.f ? min((int)(v * (float)LMOE_NBINS), LMOE_NBINS - 1) : 0;
    atomicAdd(&sh[g * LMOE_NBINS + bin], 1u);
  }
  __syncthreads();
  uint32_t* hrow = hist + (size_t)e0 * LMOE_NBINS;
  for (int i = threadIdx.x; i < g_count * LMOE_NBINS; i += blockDim.x) {
    const uint32_t v = sh[i];
    if (v) hrow[i] += v;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *ntok_acc += ntok;
}

// --------------------------------------------------------------------------- combine
// z_t = sum_i g_ti o[inv[t, i]] in rank order, fp32 accumulation; one warp per token.
template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(const T* __restrict__ o, const float* __restrict__ gates,
                                                      const int* __restrict__ inv, int ntok, int k, int l,
                                                      T* __restrict__ z) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= ntok) return;
  constexpr int VEC = 16 / sizeof(T);
  for (int v = lane; v < l / VEC; v += 32) {
    float acc[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
    for (int i = 0; i < k; ++i) {
      const float g = gates[(size_t)t * k + i];
      const int row = inv[(size_t)t * k + i];
      uint4 q = reinterpret_cast<const uint4*>(o + (size_t)row * l)[v];
      const T* e = reinterpret_cast<const T*>(&q);
#pragma unroll
      for (int j = 0; j < VEC; ++j) acc[j] = fmaf(g, to_f<T>(e[j]), acc[j]);
    }
    uint4 out;
    T* oe = reinterpret_cast<T*>(&out);
#pragma unroll
    for (int j = 0; j < VEC; ++j) oe[j] = from_f<T>(acc[j]);
    reinterpret_cast<uint4*>(z + (size_t)t * l)[v] = out;
  }
}

// --------------------------------------------------------------------------- QB update
// Block per expert: m = ceil((E-k) N / E); the crossing bin j* is the first whose cumulative
// count reaches m; q = (j* + (m - cum_{j*-1}) / cnt_{j*}) / 4096; u_e = q (+ b_e).  The row of
// the histogram is cleared afterwards.
__global__ void __launch_bounds__(256) qb_quantile_kernel(uint32_t* __restrict__ hist,
                                                          const long long* __restrict__ ntok_acc,
                                                          const float* __restrict__ bias, int E, int k,
                                                          int literal, double* __restrict__ u_out,
                                                          uint32_t* status) {
  __shared__ long long wsum[8];
  const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long N = *ntok_acc;
  if (N <= 0) return;
  long long m = ((long long)(E - k) * N + E - 1) / E;
  m = m < 1 ? 1 : (m > N ? N : m);
  uint32_t* row = hist + (size_t)e * LMOE_NBINS;
  constexpr int PER = LMOE_NBINS / 256;
  uint32_t c[PER];
  long long local = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    c[j] = row[tid * PER + j];
    local += c[j];
  }
  // inclusive scan of per-thread sums
  long long x = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long y = __shfl_up_sync(kFull, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  if (tid == 0) u_out[e] = literal ? 0.0 : (double)bias[e];
  __syncthreads();
  long long before = x - local;
  for (int w = 0; w < warp; ++w) before += wsum[w];
  if (before < m && m <= before + local) {
    long long cum = before;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      if (cum + c[j] >= m) {
        const int jstar = tid * PER + j;
        const double q = ((double)jstar + (double)(m - cum) / (double)c[j]) / (double)LMOE_NBINS;
        u_out[e] = literal ? q : q + (double)bias[e];
        break;
      }
      cum += c[j];
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < PER; ++j) row[tid * PER + j] = 0u;
}

// b_e <- b_e - beta (u_e - mean_e u); then the token count is cleared.  One block.
__global__ void __launch_bounds__(1024) qb_apply_kernel(float* __restrict__ bias, long long* ntok_acc,
                                                        const double* __restrict__ u, int E, float beta) {
  __shared__ double ws[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (*ntok_acc <= 0) return;
  double v = 0.0;
  for (int e = tid; e < E; e += blockDim.x) v += u[e];
#pragma unroll
  for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  if (lane == 0) ws[warp] = v;
  __syncthreads();
  if (warp == 0) {
    double w = ws[lane];
#pragma unroll
    for (int off = 16; off; off >>= 1) w += __shfl_xor_sync(kFull, w, off);
    if (lane == 0) ws[0] = w;
  }
  __syncthreads();
  const double mean = ws[0] / E;
  for (int e = tid; e < E; e += blockDim.x)
    bias[e] = (float)((double)bias[e] - (double)beta * (u[e] - mean));
  __syncthreads();
  if (tid == 0) *ntok_acc = 0;
}

// --------------------------------------------------------------------------- weight repacking
// out[r, c] = g[c] * w[r, c] in the storage type (gain folded into an (out, in) matrix).
template <typename T>
__global__ void fold_gain_kernel(const T* __restrict__ w, const T* __restrict__ g, int rows, int cols,
                                 T* __restrict__ out, int ld_out, int col_off) {
  const long long n = (long long)rows * cols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / cols), c = (int)(i - (long long)r * cols);
    const float gv = g ? to_f<T>(g[c]) : 1.f;
    out[(long long)r * ld_out + col_off + c] = from_f<T>(gv * to_f<T>(w[i]));
  }
}

// hi / lo bf16 pair of g[c] * w[r, c]: the product of two bf16 numbers is exact in fp32 and
// hi + lo holds it to 16 significant bits, i.e. exactly.  out is [rows, 2 cols] = [hi | lo].
__global__ void fold_gain_split_kernel(const bf16* __restrict__ w, const bf16* __restrict__ g, int rows,
                                       int cols, bf16* __restrict__ out) {
  const long long n = (long long)rows * cols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / cols), c = (int)(i - (long long)r * cols);
    const float p = __bfloat162float(g[c]) * __bfloat162float(w[i]);
    const bf16 hi = __float2bfloat16_rn(p);
    const bf16 lo = __float2bfloat16_rn(p - __bfloat162float(hi));
    out[(long long)r * 2 * cols + c] = hi;
    out[(long long)r * 2 * cols + cols + c] = lo;
  }
}

// Interleave the gate (w1) and linear (w3) projections of `groups` experts in blocks of 64 rows:
// out row (j/64)*128 + j%64 = gain * w1[j], out row (j/64)*128 + 64 + j%64 = gain * w3[j].
template <typename T>
__global__ void interleave_kernel(const T* __restrict__ w1, const T* __restrict__ w3, const T* __restrict__ g,
                                  int groups, int rows, int cols, T* __restrict__ out) {
  const long long n = (long long)groups * rows * cols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long rc = (long long)rows * cols;
    const int grp = (int)(i / rc);
    const long long rem = i - grp * rc;
    const int r = (int)(rem / cols), c = (int)(rem - (long long)r * cols);
    const float gv = g ? to_f<T>(g[c]) : 1.f;
    const long long base = (long long)grp * 2 * rc;
    const long long o1 = base + (long long)((r / 64) * 128 + (r % 64)) * cols + c;
    out[o1] = from_f<T>(gv * to_f<T>(w1[i]));
    out[o1 + 64LL * cols] = from_f<T>(gv * to_f<T>(w3[i]));
  }
}

// fp32 router weights as three bf16 parts [hi | mid | lo] per row (sum exact to 24 bits).
__global__ void split3_kernel(const float* __restrict__ w, int rows, int cols, bf16* __restrict__ out) {
  const long long n = (long long)rows * cols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / cols), c = (int)(i - (long long)r * cols);
    const float v = w[i];
    const bf16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);
    const bf16 mid = __float2bfloat16_rn(r1);
    const bf16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    bf16* o = out + (long long)r * 3 * cols + c;
    o[0] = hi;
    o[cols] = mid;
    o[2 * cols] = lo;
  }
}

}  // namespace lmoe
