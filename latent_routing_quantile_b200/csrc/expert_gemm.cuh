// Routed-expert grouped GEMMs on CTA pairs with the expert's weights as the MMA's 256-row operand.
//
// The experts' GEMMs are D_e = W_e X_e^T for each expert e: W_e its weight rows (gate and linear
// projections, or the output projection), X_e the rows of the tokens routed to it (the gathered
// latent rows, or their SwiGLU activations).  A pair of CTAs (a cluster of 2, one
// tcgen05.mma.cta_group::2 of shape 256 x N x 16 per step) computes one 256-row slice of W_e
// against up to 256 of the expert's tokens: CTA r holds weight rows [128 r, 128 r + 128) of the
// slice and tokens [r N/2, (r+1) N/2) of the tile in shared memory, and each CTA's tensor memory
// receives its own 128 weight rows against all N tokens.  N is the tile's token count rounded up
// to 32, so an expert's last tile wastes at most 31 columns (a token-row tile of 128 would waste up
// to 127 rows), and each weight slice is read once per 256 tokens.
//
// CTA = 10 warps: warp 0 issues TMA loads (no multicast) into an S-stage ring (16 KB of weights +
// up to 16 KB of tokens per stage), warp 1 of the even CTA issues the pair MMAs into one of two
// TMEM accumulators (256 columns each) and commits each stage back to both producers, warps 2-9
// drain the other accumulator: TMEM lane = weight row, column = token, so the epilogue writes the
// transpose of what it reads, 32 tokens at a time, into staged 128-byte-swizzled boxes that a TMA
// store writes to the token-major output.
//
//  XEPI_SWIGLU (gate/linear slice, K = l): in each CTA's 128 rows, lane 32q + j holds the gate
//    projection of feature 16q + (j & 15) of the CTA's 64 features when j < 16 and the linear one
//    when j >= 16 (the repacked weight order); a shuffle pairs them and out = silu(gate) * linear,
//    bf16, columns [128 slice + 64 r, +64) of act.
//  XEPI_STORE (output slice, K = h): lane = output feature; out bf16, columns
//    [256 slice + 128 r, +128) of o.
// Work items are (token tile, weight slice), slices inner, so the pairs that run at the same time
// share a token tile in L2; each tile-table entry is (expert, first row in the padded expert
// layout, valid tokens).  Every wait is bounded as in the GEMM engine.
#pragma once

#include "common.cuh"

namespace lmoe {

enum XEpilogue : int { XEPI_SWIGLU = 0, XEPI_STORE = 1 };

struct XParams {
  CUtensorMap tmW;        // weights [E * w_rows, K] bf16, box 64 x 128
  CUtensorMap tmX;        // token rows [rows, K] bf16, box 64 x 16
  CUtensorMap tmOut;      // output [rows, out_cols] bf16, box 64 x 32
  const int4* tiles;      // (expert, first row, valid tokens, 0)
  const int* num_tiles;   // entries of the table (device)
  int w_rows;             // weight rows per expert (a multiple of 256)
  int nkb;                // K / 64
  uint32_t* status;
};

constexpr int kXStages = 6;
constexpr int kXStageBytes = 32768;  // 16 KB of weight rows + at most 128 token rows x 128 bytes
constexpr int kXBoxBytes = 32 * 128;  // one staged output box: 32 tokens x 64 bf16
constexpr int kXOutOffset = kXStages * kXStageBytes;
constexpr int kXOutBytes = 2 * 2 * 2 * kXBoxBytes;  // 2 halves x 2 buffers x 2 boxes
constexpr int kXBarOffset = kXOutOffset + kXOutBytes;
constexpr int kXSmemBytes = kXBarOffset + 256 + 1024;
constexpr int kXTmemCols = 512;  // two accumulators of 256 columns

template <int EPI>
__global__ void __launch_bounds__(kTcThreads, 1) expert_gemm_kernel(const __grid_constant__ XParams p) {
  constexpr int S = kXStages;
  constexpr int kBoxes = EPI == XEPI_SWIGLU ? 1 : 2;  // output boxes per 32-token chunk and CTA
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kXBarOffset);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* bfull = tempty + 2;  // [half][buffer]: the box(es) of a chunk are written
  uint64_t* bfree = bfull + 4;   // [half][buffer]: their TMA stores have read them
  uint64_t* drain = bfree + 4;
  uint8_t* obox = smem + kXOutOffset;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int first = (int)(blockIdx.x >> 1), stride = (int)(gridDim.x >> 1);
  const int n_wt = p.w_rows / 256;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * kEpiWarps);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bfull[i], 4);  // the four lane-quarter warps of a half
      mbar_init(&bfree[i], 1);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tmW);
    tma_prefetch_desc(&p.tmX);
    tma_prefetch_desc(&p.tmOut);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kXTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // token rows, tile table and counts come from earlier kernels
  pdl_trigger();
  const int num_items = *p.num_tiles * n_wt;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs): its 128 weight rows and its half of the tokens
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      const uint64_t pol_first = l2_evict_first();
      bool ok = true;
      const uint32_t bar0 = mapa_shared(smem_u32(&full[0]), 0);
      for (int w = first; ok && w < num_items; w += stride) {
        const int tt = w / n_wt, wt = w - tt * n_wt;
        const int4 ti = p.tiles[tt];
        const int half = ((ti.z + 31) >> 5) << 4;  // N / 2, a multiple of 16
        const int wrow = ti.x * p.w_rows + wt * 256 + (int)rank * 128;
        const int xrow = ti.y + (int)rank * half;
        for (int kb = 0; kb < p.nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = smem + stage * kXStageBytes;
          uint8_t* b_dst = a_dst + 16384;
          // both CTAs' bytes complete the leader's full barrier, which expects all of them
          const uint32_t barc = bar0 + (uint32_t)(stage * 8);
          if (leader) mbar_expect_tx(&full[stage], (uint32_t)(2 * (16384 + half * 128)));
          tma_load_2d_pair_hint(a_dst, &p.tmW, barc, kb * 64, wrow, pol_first);
          for (int r = 0; r < half; r += 16) tma_load_2d_pair(b_dst + r * 128, &p.tmX, barc, kb * 64, xrow + r);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {
        for (int i = 0; i < S; ++i)
          if ((armed >> i) & 1u) mbar_drain(&full[i], (armed_parity >> i) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (the even CTA issues for the pair)
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int w = first; ok && w < num_items; w += stride, ++it) {
        const int tt = w / n_wt;
        const int nv = p.tiles[tt].z;
        const int N = ((nv + 31) >> 5) << 5;
        const uint32_t idesc = idesc_bf16_f32(N, 256);
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        for (int kb = 0; kb < p.nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * kXStageBytes);
          const uint32_t b_addr = a_addr + 16384;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_bf16_pair(d_tmem, smem_desc_sw128(a_addr + k * 32), smem_desc_sw128(b_addr + k * 32), idesc,
                             (kb | k) != 0);
          tc_commit_pair(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit_pair(&tfull[acc]);
      }
      if (!ok) {
        tc_commit_pair(drain);
        mbar_drain(drain, 0);
      }
    }
  } else {
    // ---------------- epilogue warps 2..9: TMEM lane quarter wq, half hf takes chunks c = hf, hf+2, ..
    const int wq = warp & 3;
    const int hf = (warp - 2) >> 2;
    const bool storer = wq == 2;  // warps 2 and 6 (quarter 2 of each half) issue the stores
    uint64_t* my_full = bfull + 2 * hf;
    uint64_t* my_free = bfree + 2 * hf;
    uint8_t* my_box = obox + hf * 2 * kBoxes * kXBoxBytes;
    int it = 0;
    uint32_t step = 0;
    bool ok = true;
    for (int w = first; ok && w < num_items; w += stride, ++it) {
      const int tt = w / n_wt, wt = w - tt * n_wt;
      const int4 ti = p.tiles[tt];
      const int nch = (ti.z + 31) >> 5;  // 32-token chunks
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      ok = mbar_wait(&tfull[acc], acc_phase, abort, p.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(wq * 32) << 16) + acc * 256;
      const int x0 = EPI == XEPI_SWIGLU ? wt * 128 + (int)rank * 64 : wt * 256 + (int)rank * 128;
#pragma unroll 1
      for (int c = hf; ok && c < nch; c += 2) {
        uint32_t v[32];
        tmem_ld32(tbase + c * 32, v);
        tc_wait_ld();
        const int buf = step & 1;
        const uint32_t par = (step >> 1) & 1u;
        bool good = mbar_wait(&my_free[buf], par ^ 1u, abort, p.status);
        __syncwarp();
        if (__any_sync(0xffffffffu, !good)) {
          ok = false;
          break;
        }
        uint8_t* box = my_box + buf * kBoxes * kXBoxBytes;
        if constexpr (EPI == XEPI_SWIGLU) {
          // lanes j and j ^ 16 hold the gate and linear projections of one feature: lane j < 16
          // keeps tokens 0..15 of the chunk, lane j + 16 tokens 16..31
          const bool lo = lane < 16;
          const int col = wq * 16 + (lane & 15);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t send = lo ? v[16 + i] : v[i];
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 16);
            const float g = __uint_as_float(lo ? v[i] : recv);
            const float u = __uint_as_float(lo ? recv : v[16 + i]);
            const int row = lo ? i : 16 + i;
            const bf16 a = __float2bfloat16_rn(silu_fast(g) * u);
            *reinterpret_cast<bf16*>(box + sw128_offset(row, col >> 3) + (col & 7) * 2) = a;
          }
        } else {
          const int f = wq * 32 + lane;  // output feature of this CTA's 128
          uint8_t* b = box + (f >> 6) * kXBoxBytes;
          const int col = f & 63;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            *reinterpret_cast<bf16*>(b + sw128_offset(i, col >> 3) + (col & 7) * 2) =
                __float2bfloat16_rn(__uint_as_float(v[i]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&my_full[buf]);
        if (storer) {
          good = mbar_wait(&my_full[buf], par, abort, p.status);
          __syncwarp();
          if (__any_sync(0xffffffffu, !good)) {
            ok = false;
            break;
          }
          if (lane == 0) {
#pragma unroll
            for (int bx = 0; bx < kBoxes; ++bx)
              tma_store_2d_hint(&p.tmOut, box + bx * kXBoxBytes, x0 + bx * 64, ti.y + c * 32, l2_evict_last());
            bulk_commit();
            if (step > 0) {
              bulk_wait_read<1>();  // the previous chunk's boxes have been read: that buffer is free
              mbar_arrive(&my_free[(step - 1) & 1]);
            }
          }
          __syncwarp();
        }
        ++step;
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));  // the leader's barrier
    }
    if (storer && lane == 0) bulk_wait_all();
  }

  __syncthreads();
  cluster_sync_all();  // both CTAs are done with TMEM and each other's barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kXTmemCols);
  }
  cluster_sync_all();
}

}  // namespace lmoe
