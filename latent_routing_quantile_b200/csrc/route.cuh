// Memory-bound kernels of the layer: RMSNorm reciprocal, biased top-k with gates and stable
// per-block ranks, the dispatch plan (offsets, per-block bases, grouped-GEMM tile table), the
// permutation gather, the QB score histogram, the weighted combine, and the QB update.
#pragma once

#include <climits>

#include "common.cuh"

namespace lmoe {

constexpr int kTokBlock = 32;      // tokens per routing block: one rank-mask word per expert
constexpr int kCountCopies = 32;   // per-expert counts are summed into this many copies (block % 32)
constexpr int kTileRows = 128;     // rows per grouped-GEMM M-tile
constexpr unsigned kFull = 0xffffffffu;

// --------------------------------------------------------------------------- RMSNorm
// r_t = 1 / sqrt(mean_j x_tj^2 + eps); one warp per token, squares summed in fp64.
template <typename T>
__global__ void __launch_bounds__(256) rms_kernel(const T* __restrict__ x, int ntok, int d, float eps,
                                                  float* __restrict__ r) {
  pdl_wait();
  pdl_trigger();
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
// Order-preserving map of a float to uint32 (larger float -> larger key); 0 is kept free to mark
// taken or absent experts and 1 for a NaN score, which ranks below every number.
__device__ __forceinline__ uint32_t order_key(float f) {
  // -0 + 0 = +0 under round-to-nearest (every other value is unchanged), so -0 and +0, which
  // compare equal, get one key; negative numbers have all bits flipped, the others the sign bit
  // (an XOR with the sign spread over the word, and the sign bit)
  if (f != f) return 1u;
  const uint32_t b = __float_as_uint(f + 0.0f);
  return b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
}
// Inverse of order_key for keys of numbers (>= 2).
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  return v;
}

// Inputs of the exact decision of ambiguous tokens (x == nullptr: decide every token in fp32).
struct TopkRefine {
  const void* x;      // layer input [T, d], bf16 (x_bf16) or fp32
  int x_bf16, d;
  const double* wc;   // W_comb [E, d] fp64
  const float* cz;    // router column offsets [E]
  float eps, tau;
};
constexpr int kRefineExtra = 8;  // candidates beyond the k-th that an exact decision lists
constexpr int kOverflow = 1 << 30;  // deferred-token flag: more candidates than the list holds

// The exact decision of a token whose fp32 top-k is ambiguous (two of its top k+1 biased scores
// within tau of each other, so the scores' fp32 rounding could order them either way).  Its
// candidates are its top k and every expert whose fp32 biased score lies within tau of the k-th
// (at most kRefineExtra beyond the k-th), in fp32 order.  Consecutive candidates closer than tau
// are linked; a maximal run of linked candidates is a cluster.  The fp32 error of a score is below
// tau / 2, so candidates of different clusters are in their exact order already, and only the
// members of clusters of two or more are rescored: each one's biased score is recomputed in fp64
// as the layer defines it, u = sigmoid(r * (x . W_comb[e]) + c_e) + b_e with r = 1/sqrt(mean x^2
// + eps) and W_comb the router and down-projection weights multiplied out in fp64 (the same logit
// as h W_r^T + c up to fp64 rounding), and each cluster's members are ranked among its positions by
// (u descending, expert ascending).  The whole block computes each such token's dot products
// together (one memory round trip instead of one per 32 elements), after its warps have ranked
// every other token.
//
// A token can have more experts within tau of its k-th than the candidate list holds (at most
// kRefineExtra beyond the k-th, and 32 in all): many scores that saturate the sigmoid to exactly
// 1.0f in fp32 do that, and at k = 32 the list has no room beyond the k-th at all.  Such a token
// ("overflow") is decided from every expert whose fp32 biased score lies within tau of the k-th:
// any other expert trails the k experts above it by more than tau in fp32, hence by more than
// tau / 2 exactly, so the exact top k lies among them.  Each of them is rescored in fp64 as above
// and the k best (u descending, expert ascending) are taken in that order.

// One warp per token; a block of W = 16 warps ranks kTokBlock = 32 tokens (two per warp), two
// blocks per SM (registers capped at 64).  Lane L holds the scores
// of experts L, L+32, ...; the scores of up to PF tokens are loaded before any of them is ranked,
// so their memory latency overlaps.  k rounds of: local best (larger key, then lower index),
// warp max of the keys (redux), warp min of the expert index among the lanes holding that key
// (redux); lane i keeps the i-th choice.  This is top-k of u = s + b in fp32 with ties to the
// lower expert index.  Gates are the chosen s (reloaded by the lanes that keep a choice) over
// their sum.  Each choice sets the token's bit in the expert's shared mask; the token's rank
// inside the block for that expert is the number of set bits below it, so the permutation is
// stable (token ascending) with no order-dependent atomics.  With bins != null it also stores
// each score's histogram bin, min(floor(s * 4096), 4095) as uint16, expert-major
// (bins[e * ld_bins + t]).
__host__ __device__ constexpr int topk_warps(int) { return 16; }
__host__ __device__ constexpr int topk_prefetch(int nj) { return nj <= 16 ? 2 : 1; }

template <int NJ>
// Above E = 256 the registers spill a little at the cap (364 bytes at E <= 1024), and the
// rescoring of near-tie tokens is latency-bound: at E = 896 (16384 tokens) one 8-warp block per
// SM (153 registers) took 290 us, three 8-warp blocks (80 registers) 183-273 us, two 16-warp
// blocks 243-247 us against 268-273 us for three 8-warp ones in the same runs (its 512 blocks
// fill 1.7 waves of 296 instead of 1.15 waves of 444: less of a tail).
__global__ void __launch_bounds__(32 * topk_warps(NJ), 2)
    topk_kernel(const float* __restrict__ s, const float* __restrict__ bias, int ntok, int E, int k,
                int* __restrict__ idx, float* __restrict__ gates, int* __restrict__ rank,
                int* __restrict__ blkcnt, int* __restrict__ counts32, uint16_t* __restrict__ bins, int ld_bins,
                const TopkRefine rf, uint32_t* status) {
  constexpr int W = topk_warps(NJ);
  constexpr int TPW = kTokBlock / W;  // tokens per warp
  constexpr int PF = topk_prefetch(NJ);
  // fp64 rescoring reads four elements per thread and step above E = 256 (the wide layers, whose
  // d makes the rescoring loop latency-bound)
  constexpr bool kQuad = NJ > 8;
  extern __shared__ uint32_t smem_topk[];
  uint32_t* mask = smem_topk;                                    // [E]
  uint16_t* sbins = reinterpret_cast<uint16_t*>(smem_topk + E);  // [32 tokens][E + 2] (padded rows)
  const int bpitch = E + 2;
  const int blk = blockIdx.x, t0 = blk * kTokBlock;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tokens of the block that wait for the exact decision: candidates, (token | count << 8)
  __shared__ int def_e[kTokBlock][32];
  __shared__ unsigned char def_mi[kTokBlock][32];  // candidate positions of the cluster members
  __shared__ unsigned def_lp[kTokBlock];           // bit c: candidate c is linked to candidate c-1
  __shared__ int def_info[kTokBlock];              // token | candidates << 8 | members << 16 (| kOverflow)
  __shared__ float def_thr[kTokBlock];             // overflow: the fp32 threshold u_(k) - tau
  __shared__ double ovf_u[NJ * 32];                // overflow: fp64 biased score of each candidate
  __shared__ int def_n;
  __shared__ double red[W][9];
  __shared__ double def_z[48];  // [0, 32): candidate dot products; [32, 41): first group's sums; 40: x^2
  for (int i = threadIdx.x; i < E; i += blockDim.x) mask[i] = 0;
  if (threadIdx.x == 0) def_n = 0;
  pdl_wait();
  pdl_trigger();
  float bj[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = j * 32 + lane;
    bj[j] = e < E ? bias[e] : 0.f;
  }
  __syncthreads();

  int sel_q[TPW], slot_q[TPW];
  uint32_t deferred = 0;  // tokens of this warp whose choice waits for the exact decision
  bool nan = false;
  // stores token t's choice (lane i < k holds the i-th expert): index, gate, rank-mask bit
  auto commit = [&](int t, int tl, int& my_sel) {
    float my_s = 0.f;
    if (lane < k) {
      if (my_sel < 0 || my_sel >= E) {
        set_status(status, LMOE_STATUS_BAD_INDEX);
        my_sel = 0;
      }
      my_s = s[(size_t)t * E + my_sel];
      if (my_s != my_s) my_s = 0.f;
    }
    float ssum = my_s;
#pragma unroll
    for (int off = 16; off; off >>= 1) ssum += __shfl_xor_sync(kFull, ssum, off);
    if (lane < k) {
      idx[(size_t)t * k + lane] = my_sel;
      gates[(size_t)t * k + lane] = my_s / ssum;
      atomicOr(&mask[my_sel], 1u << tl);
    }
  };
#pragma unroll
  for (int q0 = 0; q0 < TPW; q0 += PF) {
    float vq[PF][NJ];
#pragma unroll
    for (int p = 0; p < PF; ++p) {
      const int t = t0 + warp * TPW + q0 + p;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int e = j * 32 + lane;
        vq[p][j] = (t < ntok && e < E) ? s[(size_t)t * E + e] : 0.f;
      }
    }
#pragma unroll
    for (int p = 0; p < PF; ++p) {
      const int tl = warp * TPW + q0 + p, t = t0 + tl;
      sel_q[q0 + p] = -1;
      if (t >= ntok) continue;  // warp-uniform
      uint32_t key[NJ];
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int e = j * 32 + lane;
        const float v = vq[p][j];
        if (e < E) {
          nan |= (v != v);
          key[j] = order_key(v + bj[j]);
          // bin min(floor(s * 4096), 4095); the unsigned conversion takes negative scores and NaN
          // to 0 and saturates large ones
          if (bins)
            sbins[tl * bpitch + e] =
                (uint16_t)min(__float2uint_rz(v * (float)LMOE_NBINS), (unsigned)(LMOE_NBINS - 1));
        } else {
          key[j] = 0u;
        }
      }
      int my_sel = -1;
      // k rounds of selection (lane i keeps the i-th choice and its key).  With the exact decision
      // enabled, near-ties among the chosen and with the best unchosen expert (a warp max of the
      // remaining keys) then mark the token, and only a marked token takes further rounds, which
      // collect the experts within tau of the k-th (at most kRefineExtra)
      const int kmax = rf.x ? min(min(k + kRefineExtra, 32), E) : k;
      float u_k1 = 0.f, my_u = 0.f;
      bool amb = false, odd = false;  // odd: a candidate without a numeric score
      int nc = k;
      uint32_t my_key = 0u;
      // each lane keeps its best remaining key h1 (slot j1) and, while hv, the next one h2 (slot
      // j2); a round takes the warp's best h1 (ties to the lower expert), and the lane it came from
      // moves up its second, re-scanning its keys (minus the taken ones, bits of tk) only when the
      // second was used up already
      uint32_t h1 = 0u, h2 = 0u, tk = 0u;
      int j1 = 0, j2 = 0;
      bool hv = true;
      auto best_two = [&]() {
        h1 = 0u;
        h2 = 0u;
        j1 = 0;
        j2 = 0;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const uint32_t kj = ((tk >> j) & 1u) ? 0u : key[j];
          if (kj > h1) {
            h2 = h1;
            j2 = j1;
            h1 = kj;
            j1 = j;
          } else if (kj > h2) {
            h2 = kj;
            j2 = j;
          }
        }
        hv = true;
      };
      // one round: the warp's best remaining key wmax (> 0) goes to lane i
      auto take = [&](int i, uint32_t wmax) {
        const uint32_t emin = __reduce_min_sync(kFull, h1 == wmax ? (uint32_t)(j1 * 32 + lane) : 0xffffffffu);
        if ((emin & 31u) == (uint32_t)lane) {  // this lane's best was taken
          tk |= 1u << j1;
          if (hv) {
            h1 = h2;
            j1 = j2;
            hv = false;
          } else {
            best_two();
          }
        }
        if (lane == i) {
          my_sel = (int)emin;
          my_key = wmax;
        }
      };
      best_two();
      for (int i = 0; i < k; ++i) take(i, __reduce_max_sync(kFull, h1));
      if (rf.x) {
        // the chosen in order: u_i (0 for a key without a number), a near-tie between neighbours
        const bool num = my_key >= 2u;
        my_u = num ? key_value(my_key) : 0.f;
        odd = __any_sync(kFull, lane < k && !num);
        const float u_up = __shfl_up_sync(kFull, my_u, 1);
        amb = __any_sync(kFull, lane > 0 && lane < k && num && u_up - my_u < rf.tau);
        u_k1 = __shfl_sync(kFull, my_u, k - 1);
        const uint32_t nk = __reduce_max_sync(kFull, h1);  // best remaining key
        if (nk >= 2u && u_k1 - key_value(nk) < rf.tau) amb = true;
        if (amb) {  // warp-uniform: extra candidates, numbers within tau of the k-th only
          for (int i = k; i < kmax; ++i) {
            const uint32_t wmax = __reduce_max_sync(kFull, h1);
            if (wmax < 2u || !(key_value(wmax) >= u_k1 - rf.tau)) break;
            take(i, wmax);
            if (lane == i) my_u = key_value(wmax);
            nc = i + 1;
          }
        }
      }
      if (amb) {  // warp-uniform: decided by the whole block after the token loop
        int slot = 0;
        if (lane == 0) slot = atomicAdd(&def_n, 1);
        slot = __shfl_sync(kFull, slot, 0);
        // overflow: the list is full and the next expert is still within tau of the k-th
        bool ovf = false;
        if (nc == kmax && kmax < E) {
          const uint32_t nk = __reduce_max_sync(kFull, h1);
          ovf = nk >= 2u && key_value(nk) >= u_k1 - rf.tau;
        }
        if (ovf) {
          if (lane == 0) {
            def_info[slot] = tl | kOverflow;
            def_thr[slot] = u_k1 - rf.tau;
          }
          const char* xr = reinterpret_cast<const char*>(rf.x) + (size_t)t * rf.d * (rf.x_bf16 ? 2 : 4);
          for (int b = lane * 128; b < rf.d * (rf.x_bf16 ? 2 : 4); b += 32 * 128) prefetch_l2(xr + b);
          deferred |= 1u << (q0 + p);
          slot_q[q0 + p] = slot;
          continue;
        }
        // clusters: candidate c is linked to c-1 when their fp32 scores are within tau (every
        // candidate is, when one of them has no numeric score)
        const float u_up = __shfl_up_sync(kFull, my_u, 1);
        const unsigned lpm = __ballot_sync(kFull, lane > 0 && lane < nc && (odd || u_up - my_u < rf.tau));
        const unsigned mm = lpm | (lpm >> 1);  // members: linked to the previous or the next
        def_e[slot][lane] = lane < nc ? my_sel : -1;
        if ((mm >> lane) & 1u) def_mi[slot][__popc(mm & ((1u << lane) - 1u))] = (unsigned char)lane;
        if (lane == 0) {
          def_lp[slot] = lpm;
          def_info[slot] = tl | (nc << 8) | (__popc(mm) << 16);
        }
        // warm L2 with the members' fp64 weight rows and the token's input row while the warp
        // ranks its other tokens
        for (unsigned m = mm; m; m &= m - 1u) {
          const int c = __ffs(m) - 1;
          const char* row = reinterpret_cast<const char*>(rf.wc + (size_t)__shfl_sync(kFull, my_sel, c) * rf.d);
          for (int b = lane * 128; b < rf.d * 8; b += 32 * 128) prefetch_l2(row + b);
        }
        const char* xr = reinterpret_cast<const char*>(rf.x) + (size_t)t * rf.d * (rf.x_bf16 ? 2 : 4);
        for (int b = lane * 128; b < rf.d * (rf.x_bf16 ? 2 : 4); b += 32 * 128) prefetch_l2(xr + b);
        deferred |= 1u << (q0 + p);
        slot_q[q0 + p] = slot;
        continue;
      }
      if (lane >= k) my_sel = -1;
      commit(t, tl, my_sel);
      sel_q[q0 + p] = my_sel;
    }
  }
  __syncthreads();  // every deferred token is listed
  const int ndef = def_n;
  for (int di = 0; di < ndef; ++di) {  // block-uniform
    const int tl = def_info[di] & 255, nc = (def_info[di] >> 8) & 255, nm = (def_info[di] >> 16) & 255,
              t = t0 + tl;
    const size_t xoff = (size_t)t * rf.d;
    auto xval = [&](int j) -> double {
      return rf.x_bf16 ? (double)__bfloat162float(reinterpret_cast<const bf16*>(rf.x)[xoff + j])
                       : (double)reinterpret_cast<const float*>(rf.x)[xoff + j];
    };
    // x[t, 4q .. 4q+3] widened to fp64 (one 8- or 16-byte load)
    auto xquad = [&](int q, double (&xv)[4]) {
      if (rf.x_bf16) {
        const uint2 pr = reinterpret_cast<const uint2*>(reinterpret_cast<const bf16*>(rf.x) + xoff)[q];
        xv[0] = (double)__uint_as_float(pr.x << 16);
        xv[1] = (double)__uint_as_float(pr.x & 0xFFFF0000u);
        xv[2] = (double)__uint_as_float(pr.y << 16);
        xv[3] = (double)__uint_as_float(pr.y & 0xFFFF0000u);
      } else {
        const float4 f = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(rf.x) + xoff)[q];
        xv[0] = f.x;
        xv[1] = f.y;
        xv[2] = f.z;
        xv[3] = f.w;
      }
    };
    // block sums: warp shuffles, then one partial per warp in red[][u]
    auto block_sum = [&](double (&v)[9], int nv, double* out) {
#pragma unroll
      for (int u = 0; u < 9; ++u) {
        if (u < nv) {
          const double a = warp_sum_d(v[u]);
          if (lane == 0) red[warp][u] = a;
        }
      }
      __syncthreads();
      if (threadIdx.x < nv) {
        double a = 0.0;
        for (int w = 0; w < W; ++w) a += red[w][threadIdx.x];
        out[threadIdx.x] = a;
      }
      __syncthreads();
    };
    if (def_info[di] & kOverflow) {
      // every expert within tau of the k-th, rescored in fp64 (one warp per expert), then the k
      // best in order; other experts hold -inf
      double v[9];
      v[0] = 0.0;
      for (int j = threadIdx.x; j < rf.d; j += blockDim.x) {
        const double xv = xval(j);
        v[0] = fma(xv, xv, v[0]);
      }
      block_sum(v, 1, def_z + 40);
      const double r = 1.0 / sqrt(def_z[40] / rf.d + (double)rf.eps);
      const float thr = def_thr[di];
      for (int e = warp; e < E; e += W) {  // warp-uniform
        const float uf = s[(size_t)t * E + e] + bias[e];  // the fp32 biased score top-k ranked
        double u = -INFINITY;
        if (uf >= thr) {  // false for NaN
          const double* wr = rf.wc + (size_t)e * rf.d;
          double z = 0.0;
          if constexpr (kQuad) {
            for (int q = lane; q < (rf.d >> 2); q += 32) {
              double xv[4];
              xquad(q, xv);
              const double2 a = reinterpret_cast<const double2*>(wr)[2 * q];
              const double2 b = reinterpret_cast<const double2*>(wr)[2 * q + 1];
              z = fma(xv[3], b.y, fma(xv[2], b.x, fma(xv[1], a.y, fma(xv[0], a.x, z))));
            }
          } else {
            for (int j = lane; j < rf.d; j += 32) z = fma(xval(j), wr[j], z);
          }
          z = warp_sum_d(z);
          u = 1.0 / (1.0 + exp(-(r * z + (double)rf.cz[e]))) + (double)bias[e];
        }
        if (lane == 0) ovf_u[e] = u;
      }
      __syncthreads();
      if (warp == 0) {
        int sel = -1;
        for (int i = 0; i < k; ++i) {
          double bu = -INFINITY;
          int be = INT_MAX;
          for (int e = lane; e < E; e += 32) {  // ascending e: a strict > keeps the lower index
            const double uv = ovf_u[e];
            if (uv > bu) {
              bu = uv;
              be = e;
            }
          }
#pragma unroll
          for (int off = 16; off; off >>= 1) {
            const double ou = __shfl_xor_sync(kFull, bu, off);
            const int oe = __shfl_xor_sync(kFull, be, off);
            if (ou > bu || (ou == bu && oe < be)) {
              bu = ou;
              be = oe;
            }
          }
          if (lane == i) sel = be < E ? be : -1;
          __syncwarp();
          if (be < E && lane == (be & 31)) ovf_u[be] = -INFINITY;  // taken
          __syncwarp();
        }
        commit(t, tl, sel);
        def_e[di][lane] = sel;  // the owning warp reads its choice back for the ranks
      }
      __syncthreads();
      continue;
    }
    // group g sums x . W_comb[e] for members 8g..8g+7 (group 0 also sums x^2 for r)
    double v[9];
    for (int c0 = 0; c0 < nm; c0 += 8) {
      const int ng = min(8, nm - c0);
      const double* wrow[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        v[u] = 0.0;
        wrow[u] = rf.wc + (size_t)def_e[di][def_mi[di][min(c0 + u, nm - 1)]] * rf.d;
      }
      v[8] = 0.0;
      if constexpr (!kQuad) {
        for (int j = threadIdx.x; j < rf.d; j += blockDim.x) {
          const double xv = xval(j);
          v[8] = fma(xv, xv, v[8]);
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = fma(xv, wrow[u][j], v[u]);
        }
      }
      // four consecutive elements per thread and step (d is a multiple of 64): each step issues
      // the rows' 32 bytes before any product, so their latencies overlap
      for (int q = threadIdx.x; kQuad && q < (rf.d >> 2); q += blockDim.x) {
        double xv[4];
        xquad(q, xv);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[8] = fma(xv[i], xv[i], v[8]);
#pragma unroll
        for (int u0 = 0; u0 < 8; u0 += 4) {  // four rows at a time bounds the registers in flight
          if (u0 < ng) {  // block-uniform
            double2 a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (u0 + u < ng) {
                a[u] = reinterpret_cast<const double2*>(wrow[u0 + u])[2 * q];
                b[u] = reinterpret_cast<const double2*>(wrow[u0 + u])[2 * q + 1];
              }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (u0 + u < ng)
                v[u0 + u] = fma(xv[3], b[u].y, fma(xv[2], b[u].x, fma(xv[1], a[u].y, fma(xv[0], a[u].x, v[u0 + u]))));
          }
        }
      }
      if (c0 == 0) {
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (u == ng) v[u] = v[8];  // x^2 rides in slot ng of the first group's sums
        block_sum(v, ng + 1, def_z + 32);
        for (int u = 0; u < ng; ++u) {
          if (threadIdx.x == 0) def_z[u] = def_z[32 + u];
        }
        if (threadIdx.x == 0) def_z[40] = def_z[32 + ng];
        __syncthreads();
      } else {
        block_sum(v, ng, def_z + c0);
      }
    }
    const double r = 1.0 / sqrt(def_z[40] / rf.d + (double)rf.eps);
    if (warp == 0) {  // rank the candidates and store the choice like any other token's
      const int e_lane = def_e[di][lane];
      const unsigned lpm = def_lp[di], mm = lpm | (lpm >> 1);
      const bool member = (mm >> lane) & 1u;
      double my_u = 0.0;
      if (member) {
        const double z = def_z[__popc(mm & ((1u << lane) - 1u))];
        my_u = 1.0 / (1.0 + exp(-(r * z + (double)rf.cz[e_lane]))) + (double)bias[e_lane];
      }
      // a cluster starts at every candidate not linked to the previous one; a member's rank is
      // its cluster's first position plus the members of its cluster that precede it exactly
      const unsigned below = lane == 31 ? kFull : ((2u << lane) - 1u);
      const int a = 31 - __clz(~lpm & below);
      int rk = member ? a : lane;
      for (int c = 0; c < nc; ++c) {
        const double uc = __shfl_sync(kFull, my_u, c);
        const int ec = __shfl_sync(kFull, e_lane, c);
        const int ac = __shfl_sync(kFull, a, c);
        if (member && c != lane && ac == a && (uc > my_u || (uc == my_u && ec < e_lane))) ++rk;
      }
      int sel = -1;
      for (int i = 0; i < k; ++i) {
        const unsigned who = __ballot_sync(kFull, lane < nc && rk == i);
        const int src = who ? __ffs(who) - 1 : 0;
        const int ei = __shfl_sync(kFull, e_lane, src);
        if (lane == i && who) sel = ei;
      }
      commit(t, tl, sel);
      def_e[di][lane] = sel;  // the owning warp reads its choice back for the ranks
    }
    __syncthreads();
  }
#pragma unroll
  for (int q = 0; q < TPW; ++q)
    if ((deferred >> q) & 1u) sel_q[q] = def_e[slot_q[q]][lane];
  if (nan) set_status(status, LMOE_STATUS_NAN_SCORE);
  __syncthreads();

#pragma unroll
  for (int q = 0; q < TPW; ++q) {
    const int tl = warp * TPW + q, t = t0 + tl;
    if (t >= ntok) break;
    if (lane < k) rank[(size_t)t * k + lane] = __popc(mask[sel_q[q]] & ((1u << tl) - 1u));
  }
  int* ccopy = counts32 + (size_t)(blk & (kCountCopies - 1)) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = __popc(mask[e]);
    blkcnt[(size_t)blk * E + e] = c;
    if (c) atomicAdd(&ccopy[e], c);
  }
  if (bins) {
    const int nt = min(kTokBlock, ntok - t0);
    if (nt == kTokBlock) {
      // expert-major store, 16 bytes a thread: 8 tokens of one expert (4 threads per expert row of
      // the block's 32 tokens; the row starts 64-byte aligned, ld_bins being a multiple of 32)
      for (int i = threadIdx.x; i < E * 4; i += blockDim.x) {
        const int e = i >> 2, c = (i & 3) * 8;
        const uint16_t* col = sbins + c * bpitch + e;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) w[q] = (uint32_t)col[2 * q * bpitch] | ((uint32_t)col[(2 * q + 1) * bpitch] << 16);
        *reinterpret_cast<uint4*>(bins + (size_t)e * ld_bins + t0 + c) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      // the last, partial block: one token a lane
      for (int e = warp; e < E; e += W)
        if (lane < nt) bins[(size_t)e * ld_bins + t0 + lane] = sbins[lane * bpitch + e];
    }
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

// Grid: ceil(E/8) blocks of 1024 threads.  Every block sums the 32 count copies and recomputes
// the expert offsets (their exclusive scan); block 0 stores counts, offsets, the grouped-GEMM
// tile table and pad_delta;
// each block then fills blkbase[b][e] = off[e] + sum_{b' < b} blkcnt[b'][e] for its 8 experts
// (at 262144 tokens, 8192 top-k blocks: with 32 experts per block, 8 blocks did this in 86 us;
// with 8 per block, 41 us; 4 per block was no faster).
// The grouped GEMMs use a padded row layout: expert e's rows start at pad_off[e], the exclusive
// scan of counts rounded up to kTileRows, so no 128-row tile holds rows of two experts; a
// permuted row pos of expert e sits at row pos + pad_delta[e] of that layout.
constexpr int kPlanExperts = 8;
constexpr int kPlanChunks = 1024 / kPlanExperts;
__global__ void __launch_bounds__(1024) plan_kernel(const int* __restrict__ counts32, int* __restrict__ counts,
                                                    const int* __restrict__ blkcnt, int nblk, int E,
                                                    int* __restrict__ offsets, int* __restrict__ pad_delta,
                                                    int* __restrict__ blkbase, int2* __restrict__ mtiles,
                                                    int* __restrict__ num_mtiles, long long* __restrict__ load) {
  __shared__ int sh[32];
  __shared__ int s_off[1024];
  __shared__ int part[kPlanChunks][kPlanExperts + 1];
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  int c = 0;
  if (tid < E) {
    int cc[kCountCopies];  // all copies in flight at once
#pragma unroll
    for (int j = 0; j < kCountCopies; ++j) cc[j] = counts32[(size_t)j * E + tid];
#pragma unroll
    for (int j = 0; j < kCountCopies; ++j) c += cc[j];
  }
  int total;
  const int off = block_exclusive_scan_1024(c, sh, &total);
  s_off[tid] = off;
  if (blockIdx.x == 0) {
    if (tid < E) {
      offsets[tid] = off;
      counts[tid] = c;
      if (load) load[tid] += c;
    }
    if (tid == 0) offsets[E] = total;
    const int mt = (c + kTileRows - 1) / kTileRows;
    int mt_total;
    const int mt_start = block_exclusive_scan_1024(mt, sh, &mt_total);
    const int poff = mt_start * kTileRows;  // padded offset of this expert
    if (tid < E) pad_delta[tid] = poff - off;
    // entry: x = expert | (valid rows of the tile << 16), y = first row in the padded layout
    for (int j = 0; j < mt; ++j)
      mtiles[mt_start + j] = make_int2(tid | (min(kTileRows, c - j * kTileRows) << 16), poff + j * kTileRows);
    if (tid == 0) *num_mtiles = mt_total;

  }
  __syncthreads();
  // block bases: this block's kPlanExperts experts, the top-k blocks cut into kPlanChunks chunks
  // (a warp reads 8 experts' counts of 4 top-k blocks: whole 32-byte sectors)
  const int tx = tid % kPlanExperts, ty = tid / kPlanExperts;
  const int e = blockIdx.x * kPlanExperts + tx;
  const int chunk = (nblk + kPlanChunks - 1) / kPlanChunks;
  const int b0 = ty * chunk, b1 = min(nblk, b0 + chunk);
  // the chunk's counts are loaded in batches of 8 independent loads (one latency per batch);
  // chunks of up to 8 blocks keep them in registers for the second pass
  constexpr int kBatch = 8;
  int keep[kBatch];
  int sum = 0;
  if (e < E)
    for (int b = b0; b < b1; b += kBatch) {
      int v[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) v[i] = (b + i < b1) ? blkcnt[(size_t)(b + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        sum += v[i];
        keep[i] = v[i];
      }
    }
  part[ty][tx] = sum;
  __syncthreads();
  if (e < E) {
    int run = s_off[e];
    for (int q = 0; q < ty; ++q) run += part[q][tx];
    for (int b = b0; b < b1; b += kBatch) {
      int v[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i)
        v[i] = chunk <= kBatch ? keep[i] : ((b + i < b1) ? blkcnt[(size_t)(b + i) * E + e] : 0);
#pragma unroll
      for (int i = 0; i < kBatch; ++i)
        if (b + i < b1) {
          blkbase[(size_t)(b + i) * E + e] = run;
          run += v[i];
        }
    }
  }
}

// --------------------------------------------------------------------------- gather
// One warp per (token, slot): its permuted row pos = blkbase[block][e] + rank; records
// perm[pos] = token and inv[(t, i)] = pos, and copies the token's latent row into the padded
// expert layout at row prow[(t, i)] = pos + pad_delta[e] (prow and dst may be null: then only the
// permutation is written).
constexpr int kGatherPairs = 4;  // (token, slot) pairs per warp, their row copies issued together

template <typename T>
__global__ void __launch_bounds__(256) gather_kernel(const T* __restrict__ src, int ld_src, int l,
                                                     const int* __restrict__ idx, const int* __restrict__ rank,
                                                     const int* __restrict__ blkbase,
                                                     const int* __restrict__ pad_delta, int ntok, int E, int k,
                                                     int* __restrict__ perm, int* __restrict__ inv,
                                                     int* __restrict__ prow, T* __restrict__ dst,
                                                     int4* __restrict__ clear, int nclear, uint32_t* status) {
  pdl_wait();
  pdl_trigger();
  // the top-k count copies were last read by the plan kernel: the last block clears them for
  // the next routing (nclear 16-byte words)
  if (clear && blockIdx.x == gridDim.x - 1)
    for (int i = threadIdx.x; i < nclear; i += blockDim.x) clear[i] = make_int4(0, 0, 0, 0);
  const int lane = threadIdx.x & 31;
  const int pair0 = (blockIdx.x * 8 + (threadIdx.x >> 5)) * kGatherPairs;
  const int npairs = ntok * k;
  // lanes 0..3 resolve one pair each
  int t = -1, prow_v = 0;
  if (lane < kGatherPairs && pair0 + lane < npairs) {
    const int pair = pair0 + lane;
    const int tt = pair / k, e = idx[pair];
    if (e < 0 || e >= E) {
      set_status(status, LMOE_STATUS_BAD_INDEX);
    } else {
      const int pos = blkbase[(size_t)(tt / kTokBlock) * E + e] + rank[pair];
      if (pos < 0 || pos >= npairs) {
        set_status(status, LMOE_STATUS_BAD_INDEX);
      } else {
        t = tt;
        prow_v = pad_delta ? pos + pad_delta[e] : pos;
        inv[pair] = pos;
        perm[pos] = tt;
        if (prow) prow[pair] = prow_v;
      }
    }
  }
  if (!dst) return;
  constexpr int VEC = 16 / sizeof(T);
  int ts[kGatherPairs], rows[kGatherPairs];
#pragma unroll
  for (int j = 0; j < kGatherPairs; ++j) {
    ts[j] = __shfl_sync(kFull, t, j);
    rows[j] = __shfl_sync(kFull, prow_v, j);
  }
  for (int v = lane; v < l / VEC; v += 32) {
    uint4 q[kGatherPairs];
#pragma unroll
    for (int j = 0; j < kGatherPairs; ++j)
      if (ts[j] >= 0) q[j] = reinterpret_cast<const uint4*>(src + (size_t)ts[j] * ld_src)[v];
#pragma unroll
    for (int j = 0; j < kGatherPairs; ++j)
      if (ts[j] >= 0) reinterpret_cast<uint4*>(dst + (size_t)rows[j] * l)[v] = q[j];
  }
}

// --------------------------------------------------------------------------- QB histogram
// Block per expert: counts that expert's uint16 bins (written expert-major by the top-k kernel)
// in a shared 4096-bin histogram, then adds it into the expert's global row, which no other
// block touches.  Thread i owns bins [8i, 8i + 8) of the row; it loads them before counting so
// their latency overlaps the counting.  Block 0 adds T to the recorded token count.
constexpr int kHistThreads = LMOE_NBINS / 8;

__global__ void __launch_bounds__(kHistThreads) hist_kernel(const uint16_t* __restrict__ bins, int ld_bins,
                                                            int ntok, uint32_t* __restrict__ hist,
                                                            long long* ntok_acc) {
  __shared__ __align__(16) uint32_t sh[LMOE_NBINS];
  const int e = blockIdx.x;
  for (int i = threadIdx.x; i < LMOE_NBINS; i += blockDim.x) sh[i] = 0;
  pdl_wait();
  pdl_trigger();
  uint4* hrow4 = reinterpret_cast<uint4*>(hist + (size_t)e * LMOE_NBINS) + 2 * threadIdx.x;
  uint4 g0 = hrow4[0], g1 = hrow4[1];
  __syncthreads();
  const uint16_t* row = bins + (size_t)e * ld_bins;
  const int nvec = ntok / 8;  // ld_bins is a multiple of 32, so rows are 16-byte aligned
  const uint4* row4 = reinterpret_cast<const uint4*>(row);
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    const uint4 q = row4[v];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      atomicAdd(&sh[w[j] & 0xFFFFu], 1u);
      atomicAdd(&sh[w[j] >> 16], 1u);
    }
  }
  for (int t = nvec * 8 + threadIdx.x; t < ntok; t += blockDim.x) atomicAdd(&sh[row[t]], 1u);
  __syncthreads();
  const uint4 a0 = reinterpret_cast<const uint4*>(sh)[2 * threadIdx.x];
  const uint4 a1 = reinterpret_cast<const uint4*>(sh)[2 * threadIdx.x + 1];
  g0.x += a0.x; g0.y += a0.y; g0.z += a0.z; g0.w += a0.w;
  g1.x += a1.x; g1.y += a1.y; g1.z += a1.z; g1.w += a1.w;
  hrow4[0] = g0;
  hrow4[1] = g1;
  if (e == 0 && threadIdx.x == 0) *ntok_acc += ntok;
}

// --------------------------------------------------------------------------- combine
// z_t = sum_i g_ti o[prow[t, i]] in rank order (prow: the pair's row in the padded expert layout),
// fp32 accumulation; one warp per token.  The row loads of G slots are issued together before
// their FMAs (G >= k where possible: the launch picks the smallest of 2, 4, 6, 8 that covers k),
// and G sizes the registers, so small k keeps more warps resident.
template <typename T, int G>
__global__ void __launch_bounds__(256, (G <= 6 && sizeof(T) == 2) ? 4 : 3) combine_kernel(const T* __restrict__ o, const float* __restrict__ gates,
                                                         const int* __restrict__ prow, int ntok, int k, int l,
                                                         T* __restrict__ z) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= ntok) return;
  constexpr int VEC = 16 / sizeof(T);
  // lane i < k holds slot i's gate and row
  const float g_l = lane < k ? gates[(size_t)t * k + lane] : 0.f;
  const int r_l = lane < k ? prow[(size_t)t * k + lane] : 0;
  // every lane runs every trip (a row narrower than 32 vectors leaves some lanes idle), so the
  // shuffles that hand out slot i's gate and row always see the lane that holds them
  const int nvec = l / VEC;
  for (int v0 = 0; v0 < nvec; v0 += 32) {
    const int v = v0 + lane;
    const bool act = v < nvec;
    float acc[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
    for (int i0 = 0; i0 < k; i0 += G) {
      uint4 q[G];
      float g[G];
#pragma unroll
      for (int u = 0; u < G; ++u) {
        const int i = i0 + u;
        const int row = __shfl_sync(kFull, r_l, i & 31);
        g[u] = __shfl_sync(kFull, g_l, i & 31);
        if (act && i < k) q[u] = reinterpret_cast<const uint4*>(o + (size_t)row * l)[v];
      }
#pragma unroll
      for (int u = 0; u < G; ++u) {
        if (i0 + u >= k) break;
        const T* e = reinterpret_cast<const T*>(&q[u]);
#pragma unroll
        for (int j = 0; j < VEC; ++j) acc[j] = fmaf(g[u], to_f<T>(e[j]), acc[j]);
      }
    }
    if (!act) continue;
    uint4 out;
    T* oe = reinterpret_cast<T*>(&out);
#pragma unroll
    for (int j = 0; j < VEC; ++j) oe[j] = from_f<T>(acc[j]);
    reinterpret_cast<uint4*>(z + (size_t)t * l)[v] = out;
  }
}

// --------------------------------------------------------------------------- QB update
// One kernel, block per expert, for both bias rules.  The statistics are the accumulated
// histogram rows (when hist_live; otherwise they are known to be zero and are not touched) plus,
// when pend_T > 0, the bins of the last recorded forward that no kernel has counted yet (bins
// [E, ld_bins], pend_T tokens): N = *ntok_acc + pend_T; with N == 0 the bias is left unchanged.
//  QB (sign_rule == 0): block e counts its expert's row into a shared 4096-bin histogram, finds
//   m = ceil((E-k) N / E), the crossing bin j* (the first whose cumulative count reaches m) and
//   q = (j* + (m - cum_{j*-1}) / cnt_{j*}) / 4096, then u_e = q (+ b_e unless literal).  The last
//   block to finish (a device-wide counter) computes mean_e u and applies
//   b_e <- b_e - beta (u_e - mean) to every expert.
//  Sign rule (sign_rule == 1): the last block applies b_e <- b_e + beta sign(mean load - load_e),
//   the sign taken in integers as sign(sum_e' load_e' - E load_e).
// Either way the accumulated rows are cleared, and the last block clears N, the loads and the
// counter: an update consumes all statistics recorded since the previous one.
constexpr int kQbThreads = 256;

__global__ void __launch_bounds__(kQbThreads) qb_update_kernel(uint32_t* __restrict__ hist, long long* ntok_acc,
                                                               long long* __restrict__ load,
                                                               float* __restrict__ bias, int E, int k, int literal,
                                                               int sign_rule, float beta, double* __restrict__ u_buf,
                                                               unsigned int* done_counter,
                                                               const uint16_t* __restrict__ bins, int ld_bins,
                                                               int pend_T, int hist_live, uint32_t* status) {
  __shared__ __align__(16) uint32_t sh[LMOE_NBINS];
  __shared__ long long wsum[8];
  __shared__ double wd[8];
  __shared__ double u_sh;
  __shared__ bool last;
  const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_trigger();
  const long long N = *ntok_acc + (long long)pend_T;
  uint4* row4 = reinterpret_cast<uint4*>(hist + (size_t)e * LMOE_NBINS);
  constexpr int PER = LMOE_NBINS / kQbThreads;  // 16 bins per thread, 4 x uint4
  if (N <= 0) {  // nothing recorded: the bias stays; rows set without tokens are dropped
    if (hist_live)
      for (int j = 0; j < PER / 4; ++j) row4[tid * (PER / 4) + j] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  if (!sign_rule) {
    // shared histogram = accumulated row + the pending bins of this expert
    uint4* sh4 = reinterpret_cast<uint4*>(sh);
#pragma unroll
    for (int j = 0; j < PER / 4; ++j)
      sh4[tid * (PER / 4) + j] = hist_live ? row4[tid * (PER / 4) + j] : make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    if (pend_T > 0) {
      const uint16_t* brow = bins + (size_t)e * ld_bins;
      const int nvec = pend_T / 8;  // ld_bins is a multiple of 32, so rows are 16-byte aligned
      for (int v = tid; v < nvec; v += kQbThreads) {
        const uint4 q = reinterpret_cast<const uint4*>(brow)[v];
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          atomicAdd(&sh[w[j] & 0xFFFFu], 1u);
          atomicAdd(&sh[w[j] >> 16], 1u);
        }
      }
      for (int t = nvec * 8 + tid; t < pend_T; t += kQbThreads) atomicAdd(&sh[brow[t]], 1u);
      __syncthreads();
    }
    long long m = ((long long)(E - k) * N + E - 1) / E;
    m = m < 1 ? 1 : (m > N ? N : m);
    uint32_t c[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) c[j] = sh[tid * PER + j];
    long long local = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) local += c[j];
    long long x = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long y = __shfl_up_sync(kFull, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    if (tid == 0) u_sh = literal ? 0.0 : (double)bias[e];  // only if no crossing is found
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
          u_sh = literal ? q : q + (double)bias[e];
          break;
        }
        cum += c[j];
      }
    }
    __syncthreads();
  }
  if (hist_live) {
#pragma unroll
    for (int j = 0; j < PER / 4; ++j) row4[tid * (PER / 4) + j] = make_uint4(0u, 0u, 0u, 0u);
  }
  // thread 0 publishes u_e, then counts finished blocks (the cleared rows are read only by later
  // kernels, so they need no fence)
  if (tid == 0) {
    if (!sign_rule) u_buf[e] = u_sh;
    __threadfence();
    last = (atomicAdd(done_counter, 1u) == (unsigned)(E - 1));
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (sign_rule) {
    long long v = 0;
    for (int i = tid; i < E; i += blockDim.x) v += __ldcg(&load[i]);
#pragma unroll
    for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
    if (lane == 0) wsum[warp] = v;
    __syncthreads();
    long long tot = 0;
    for (int w = 0; w < 8; ++w) tot += wsum[w];
    for (int i = tid; i < E; i += blockDim.x) {
      const long long diff = tot - (long long)E * __ldcg(&load[i]);
      const float dir = diff > 0 ? 1.f : (diff < 0 ? -1.f : 0.f);
      bias[i] = __fadd_rn(bias[i], beta * dir);
    }
  } else {
    double v = 0.0;
    for (int i = tid; i < E; i += blockDim.x) v += __ldcg(&u_buf[i]);
#pragma unroll
    for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
    if (lane == 0) wd[warp] = v;
    __syncthreads();
    double tot = 0.0;
    for (int w = 0; w < 8; ++w) tot += wd[w];
    const double mean = tot / E;
    for (int i = tid; i < E; i += blockDim.x)
      bias[i] = (float)((double)bias[i] - (double)beta * (__ldcg(&u_buf[i]) - mean));
  }
  for (int i = tid; i < E; i += blockDim.x) load[i] = 0;
  if (tid == 0) {
    *ntok_acc = 0;
    *done_counter = 0u;
  }
}

// --------------------------------------------------------------------------- weight repacking
// W_comb[e, j] = g_j * sum_i W_r[e, i] W_down[i, j] in fp64 (g = null: gain one): the router logit
// as a single map of x (z = r * x W_comb^T + c), for the exact decision of ambiguous tokens.
// Grid (ceil(d / 256), E), one output per thread.
template <typename T>
__global__ void __launch_bounds__(256) combine_router_kernel(const float* __restrict__ w_r,
                                                             const T* __restrict__ w_down, const T* __restrict__ g,
                                                             int l, int d, double* __restrict__ wc) {
  const int e = blockIdx.y, j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  double acc = 0.0;
  for (int i = 0; i < l; ++i)
    acc = fma((double)w_r[(size_t)e * l + i], (double)to_f<T>(w_down[(size_t)i * d + j]), acc);
  wc[(size_t)e * d + j] = g ? acc * (double)to_f<T>(g[j]) : acc;
}

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

// fp32 values as three bf16 parts hi, mid, lo (hi = bf16(v), mid = bf16(v - hi), lo = bf16(v - hi
// - mid); their sum is v to fp32's 24 bits): out[r, col_off + part * cols + c] for v = g[c] w[r, c]
// (g = null: v = w[r, c]; the product rounded to fp32 once), ld_out elements per output row.
__global__ void split3_kernel(const float* __restrict__ w, const float* __restrict__ g, int rows, int cols,
                              bf16* __restrict__ out, int ld_out, int col_off) {
  pdl_wait();
  pdl_trigger();
  const long long n = (long long)rows * cols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / cols), c = (int)(i - (long long)r * cols);
    const float v = g ? g[c] * w[i] : w[i];
    const bf16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);
    const bf16 mid = __float2bfloat16_rn(r1);
    const bf16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    bf16* o = out + (long long)r * ld_out + col_off + c;
    o[0] = hi;
    o[cols] = mid;
    o[2 * cols] = lo;
  }
}

// Gate (w1) and linear (w3) rows of `groups` fp32 matrices [groups, rows, cols] interleaved in
// blocks of 64 as interleave_kernel does, each row (times the gain g, when given) split into
// three bf16 parts along cols: out [groups * 2 rows, 3 cols].
__global__ void interleave_split3_kernel(const float* __restrict__ w1, const float* __restrict__ w3,
                                         const float* __restrict__ g, int groups, int rows, int cols,
                                         bf16* __restrict__ out) {
  const long long n = (long long)groups * rows * cols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long rc = (long long)rows * cols;
    const int grp = (int)(i / rc);
    const long long rem = i - grp * rc;
    const int r = (int)(rem / cols), c = (int)(rem - (long long)r * cols);
    const long long orow = (long long)grp * 2 * rows + (r / 64) * 128 + (r % 64);
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const float v = (g ? g[c] : 1.f) * (which ? w3[i] : w1[i]);
      const bf16 hi = __float2bfloat16_rn(v);
      const float r1 = v - __bfloat162float(hi);
      const bf16 mid = __float2bfloat16_rn(r1);
      const bf16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
      bf16* o = out + (orow + which * 64) * 3 * cols + c;
      o[0] = hi;
      o[cols] = mid;
      o[2 * cols] = lo;
    }
  }
}

}  // namespace lmoe
