// Fused RMSNorm + latent down-projection + sigmoid router for sm_100a (l <= 256, E <= 256).
//
// One CTA, or a cluster of ns = 2 CTAs, per 128-token tile (persistent over tiles), 10 warps: warp
// 0 issues TMA loads into a 4-stage shared-memory ring, warp 1 issues tcgen05.mma, warps 2-9 are
// the epilogue.  With ns = 2 (few tiles: twice the SMs at work) CTA rank r of the cluster
// computes columns [r l/2, (r+1) l/2) of h and experts [r E/2, (r+1) E/2) of s: each loads half
// of W_down and of the router weights, and both read all of h back in phase C, so phase C waits
// until both CTAs' h stores have completed (each storer arrives on both CTAs' barrier).
//   Phase A  h_acc[128, l] = x_tile W_down'^T in TMEM columns [0, l).  While each x stage sits in
//            shared memory the epilogue warps add up the squares of their rows (a sum does not
//            care about the 128-byte swizzle order), so r_t = 1/sqrt(mean x^2 + eps) costs no
//            extra pass over x.
//   Phase B  epilogue: h = r_t h_acc, stored as hi | mid | lo bf16 parts (hi = bf16(h) feeds the
//            routed experts; the three parts hold fp32's 24 bits for the router), r_t stored for
//            the shared expert.  The parts leave by TMA stores (staged 16 KB boxes, as in the GEMM
//            engine), stay in L2 and are loaded back by TMA once the stores have completed.
//   Phase C  z[128, E] = six bf16 x bf16 products of the h parts with the hi/mid/lo parts of the
//            fp32 router weights.  When E/ns <= l/ns (the usual case) phase C walks K chunk by
//            chunk: the three h parts and the three weight parts of a 64-column chunk are loaded
//            once (three ring stages) and feed all six products; hi x hi accumulates in TMEM
//            columns [l/ns, l/ns + E/ns) and the five smaller products in columns [0, E/ns) (h's
//            accumulator, free once phase B has read it), so the small terms are summed among
//            themselves before phase D adds the two.  Otherwise it walks product by product
//            (smallest first) into one accumulator, reloading parts.
//   Phase D  epilogue: s = sigmoid(z + c), fp32.
// Every wait is bounded as in the GEMM engine; a wait that expires sets LMOE_STATUS_WATCHDOG and
// the CTA winds down.
#pragma once

#include "common.cuh"

namespace lmoe {

struct K1Params {
  CUtensorMap tm_s;   // s [Tm, E] fp32, box 32 x 128 (output)
  CUtensorMap tm_x;   // x [T, d], box 64 x 128
  CUtensorMap tm_wd;  // W_down' [l, d] or [l, 2d] (hi | lo when the gain is not one), box 64 x l/ns
  CUtensorMap tm_hx;  // h parts [Tm, 3l], box 64 x 128 (output, then A of phase C)
  CUtensorMap tm_wr;  // router parts [E, 3l], box 64 x E/ns
  int T, d, l, E;
  int ns;             // CTAs per tile: 1, or 2 (launched as clusters of 2; l % 128 == 0, E % 64 == 0)
  int wd_segments;    // 1, or 2 when W_down' is split into hi | lo
  float eps;
  float* r;           // out: [T]
  const float* c;     // router column offsets [E]
  uint32_t* status;
};

// A stage holds a 16 KB x (or h part) box and the B rows of one k-block (at most 256 x 128 bytes);
// the ring gets as many stages as fit in 192 KB: 4 when B has 256 rows, 6 with 128 rows.
constexpr int kK1RingBytes = 192 * 1024;
constexpr int kK1MaxStages = 8;
constexpr int kK1OutOffset = kK1RingBytes;  // two 16 KB output boxes
constexpr int kK1BarOffset = kK1OutOffset + 2 * 16384;
constexpr int kK1SmemBytes = kK1BarOffset + 384 + 1024 + 1024;  // barriers, RMS partials, alignment slack

__global__ void __launch_bounds__(kTcThreads, 1) k1_kernel(const __grid_constant__ K1Params p) {
  const int brows = (p.l > p.E ? p.l : p.E) / p.ns;  // B rows per stage
  const int stage_bytes = 16384 + brows * 128;
  int S = kK1RingBytes / stage_bytes;
  S = S > kK1MaxStages ? kK1MaxStages : S;  // 3 x S + 13 barriers and two words fit in 384 bytes
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kK1BarOffset);
  uint64_t* empty = full + S;
  uint64_t* rmsd = empty + S;
  uint64_t* tfullA = rmsd + S;
  uint64_t* tempA = tfullA + 1;
  uint64_t* hxr = tempA + 1;
  uint64_t* tfullC = hxr + 1;
  uint64_t* tempC = tfullC + 1;
  uint64_t* rmsx = tempC + 1;  // both halves of every row's sum of squares are in rms_part
  uint64_t* bfull = rmsx + 1;  // output box written by all epilogue warps
  uint64_t* bfree = bfull + 2; // output box read by its TMA store
  uint64_t* drain = bfree + 2;
  uint64_t* hxs = drain + 1;   // every epilogue warp has staged its h parts in the ring
  uint64_t* sds = hxs + 1;     // every epilogue warp has staged its scores in the ring (last tile)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sds + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* rms_part = reinterpret_cast<float*>(smem + kK1BarOffset + 384);  // [2][128]
  uint8_t* obox = smem + kK1OutOffset;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ns = p.ns;
  const uint32_t rank = ns == 2 ? cluster_ctarank() : 0u;
  const int lh = p.l / ns, eh = p.E / ns;  // this CTA's columns of h and of s
  const int first = (int)blockIdx.x / ns, stride = (int)gridDim.x / ns;
  const uint32_t tmem_cols = ns == 2 ? 256u : 512u;
  const int nkd = p.d / 64, nkl = p.l / 64;
  const bool dual = eh <= lh;  // phase C chunk-major with a second accumulator (see above)
  const int nkbA = nkd * p.wd_segments, nkbC = (dual ? 3 : 6) * nkl;
  const uint32_t bytesA = 16384u + (uint32_t)lh * 128u, bytesC = 16384u + (uint32_t)eh * 128u;
  // the six significant products of (hi, mid, lo) parts, smallest first, as (A part, B part):
  // (mid, mid), (lo, hi), (hi, lo), (mid, hi), (hi, mid), (hi, hi); three bits per product
  constexpr uint32_t kProdA = 1u | (2u << 3) | (0u << 6) | (1u << 9) | (0u << 12) | (0u << 15);
  constexpr uint32_t kProdB = 1u | (0u << 3) | (2u << 6) | (0u << 9) | (1u << 12) | (0u << 15);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&rmsd[i], kEpiWarps);
    }
    mbar_init(tfullA, 1);
    mbar_init(tempA, kEpiWarps);
    mbar_init(hxr, ns);  // the storer of every CTA of the tile, once its h parts have landed
    mbar_init(tfullC, 1);
    mbar_init(tempC, kEpiWarps);
    mbar_init(rmsx, kEpiWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bfull[i], kEpiWarps);
      mbar_init(&bfree[i], 1);
    }
    mbar_init(drain, 1);
    mbar_init(hxs, kEpiWarps);
    mbar_init(sds, kEpiWarps);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_x);
    tma_prefetch_desc(&p.tm_wd);
    tma_prefetch_desc(&p.tm_hx);
    tma_prefetch_desc(&p.tm_wr);
    tma_prefetch_desc(&p.tm_s);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (ns == 2) cluster_sync_all();  // the peer's barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // x may come from an earlier kernel; hx and s are read by earlier ones
  pdl_trigger();
  const int num_tiles = (p.T + 127) / 128;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;     // full-barrier phases in flight, for the abort drain
      uint32_t rms_pend = 0, rms_par = 0;    // stages whose x must still be read for the RMS
      uint32_t rms_cnt = 0;                  // per-stage use counts (bit = parity) of the rmsd barrier
      bool ok = true;
      int it = 0;
      for (int tile = first; ok && tile < num_tiles; tile += stride, ++it) {
        const int row0 = tile * 128;
        for (int kb = 0; ok && kb < nkbA + nkbC; ++kb) {
          if (kb == nkbA) {  // every CTA's h parts are stored
            if (!mbar_wait(hxr, it & 1, abort, p.status, kWaitLimitCycles, ns == 2)) {
              ok = false;
              break;
            }
            fence_proxy_async_global();
          }
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          if ((rms_pend >> stage) & 1u) {
            if (!mbar_wait(&rmsd[stage], (rms_par >> stage) & 1u, abort, p.status)) {
              ok = false;
              break;
            }
            rms_pend &= ~(1u << stage);
          }
          uint8_t* a_dst = smem + stage * stage_bytes;
          uint8_t* b_dst = a_dst + 16384;
          if (kb < nkbA) {
            const int seg = kb / nkd, kk = kb - seg * nkd;
            mbar_expect_tx(&full[stage], bytesA);
            tma_load_2d(a_dst, &p.tm_x, &full[stage], kk * 64, row0);
            tma_load_2d(b_dst, &p.tm_wd, &full[stage], seg * p.d + kk * 64, (int)rank * lh);
            if (seg == 0) {
              rms_pend |= 1u << stage;
              rms_par = (rms_par & ~(1u << stage)) | (((rms_cnt >> stage) & 1u) << stage);
              rms_cnt ^= 1u << stage;
            }
          } else {
            int kk, pa, pb;
            if (dual) {  // chunk kk, part pa = pb of h and of the router weights
              kk = (kb - nkbA) / 3;
              pa = pb = (kb - nkbA) - 3 * kk;
            } else {     // product pr, chunk kk
              const int pr = (kb - nkbA) / nkl;
              kk = (kb - nkbA) - pr * nkl;
              pa = (int)((kProdA >> (3 * pr)) & 7u);
              pb = (int)((kProdB >> (3 * pr)) & 7u);
            }
            mbar_expect_tx(&full[stage], bytesC);
            tma_load_2d(a_dst, &p.tm_hx, &full[stage], pa * p.l + kk * 64, row0);
            tma_load_2d(b_dst, &p.tm_wr, &full[stage], pb * p.l + kk * 64, (int)rank * eh);
          }
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok)
        for (int i = 0; i < S; ++i)
          if ((armed >> i) & 1u) mbar_drain(&full[i], (armed_par >> i) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idescA = idesc_bf16_f32(lh), idescC = idesc_bf16_f32(eh);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = first; ok && tile < num_tiles; tile += stride, ++it) {
        for (int ph = 0; ok && ph < 2; ++ph) {
          const int nkb = ph == 0 ? nkbA : nkbC;
          if (!mbar_wait(ph == 0 ? tempA : tempC, (it & 1) ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          // dual phase C writes columns [0, E/ns): the epilogue must have read h out of them, and
          // the next phase A must wait until phase D has read the small products
          if (dual && !mbar_wait(ph == 0 ? tempC : tempA, ph == 0 ? (it & 1) ^ 1u : (it & 1), abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (ph == 1 && dual) {
            const uint32_t d_big = tmem_base + (uint32_t)lh, d_small = tmem_base;
            for (int kk = 0; ok && kk < nkl; ++kk) {
              uint32_t a_addr[3], b_addr[3];
              int st3[3];
#pragma unroll
              for (int q = 0; q < 3; ++q) {
                if (!mbar_wait(&full[stage], phase, abort, p.status)) {
                  ok = false;
                  break;
                }
                a_addr[q] = smem_u32(smem + stage * stage_bytes);
                b_addr[q] = a_addr[q] + 16384;
                st3[q] = stage;
                if (++stage == S) {
                  stage = 0;
                  phase ^= 1u;
                }
              }
              if (!ok) break;
              tc_fence_after();
#pragma unroll
              for (int pr = 0; pr < 5; ++pr) {  // (mid,mid) (lo,hi) (hi,lo) (mid,hi) (hi,mid)
                const int pa = (int)((kProdA >> (3 * pr)) & 7u), pb = (int)((kProdB >> (3 * pr)) & 7u);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  tc_mma_bf16(d_small, smem_desc_sw128(a_addr[pa] + k * 32), smem_desc_sw128(b_addr[pb] + k * 32),
                              idescC, (kk | pr | k) != 0);
              }
#pragma unroll
              for (int k = 0; k < 4; ++k)
                tc_mma_bf16(d_big, smem_desc_sw128(a_addr[0] + k * 32), smem_desc_sw128(b_addr[0] + k * 32), idescC,
                            (kk | k) != 0);
#pragma unroll
              for (int q = 0; q < 3; ++q) tc_commit(&empty[st3[q]]);
            }
            if (ok) tc_commit(tfullC);
            continue;
          }
          const uint32_t d_tmem = tmem_base + (ph == 0 ? 0u : (uint32_t)lh);
          const uint32_t idesc = ph == 0 ? idescA : idescC;
          for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + stage * stage_bytes);
            const uint32_t b_addr = a_addr + 16384;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_bf16(d_tmem, smem_desc_sw128(a_addr + k * 32), smem_desc_sw128(b_addr + k * 32), idesc,
                          (kb | k) != 0);
            tc_commit(&empty[stage]);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (ok) tc_commit(ph == 0 ? tfullA : tfullC);
        }
      }
      if (!ok) {
        tc_commit(drain);
        mbar_drain(drain, 0);
      }
    }
  } else {
    // ---------------- epilogue warps 2..9: TMEM lane quarter (warp % 4), column half (warp-2)/4
    const int wq = warp & 3, half_id = (warp - 2) >> 2;
    const int rl = wq * 32 + lane;  // row of the tile this thread owns
    const bool storer = (warp == 2);
    int stage = 0;
    uint32_t phase = 0;
    uint32_t step = 0;
    bool ok = true;
    int it = 0;
    // Writes this thread's 64 bytes into the current output box, then (storer) stores the box.
    auto emit = [&](const uint32_t (&w)[16], const CUtensorMap* map, int x, int y) -> bool {
      const int buf = step & 1;
      const uint32_t par = (step >> 1) & 1u;
      bool good = mbar_wait(&bfree[buf], par ^ 1u, abort, p.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !good)) return false;
      uint8_t* box = obox + buf * 16384;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(box + sw128_offset(rl, half_id * 4 + q)) =
            make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bfull[buf]);
      if (storer) {
        good = mbar_wait(&bfull[buf], par, abort, p.status);
        __syncwarp();
        if (__any_sync(0xffffffffu, !good)) return false;
        if (lane == 0) {
          tma_store_2d(map, box, x, y);
          bulk_commit();
          if (step > 0) {
            bulk_wait_read<1>();
            mbar_arrive(&bfree[(step - 1) & 1]);
          }
        }
        __syncwarp();
      }
      ++step;
      return true;
    };
    // router column offsets: lane m keeps c[j*32 + m] for every 32-column step j (E <= 256), loaded
    // once, long before phase D uses them
    float c_lane[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) c_lane[j] = (j * 32 + lane < eh) ? p.c[(int)rank * eh + j * 32 + lane] : 0.f;
    for (int tile = first; ok && tile < num_tiles; tile += stride, ++it) {
      const int row0 = tile * 128, row = row0 + rl;
      const bool valid = row < p.T;
      // phase A: squares of this row's half of every x stage (first W_down segment only)
      double ss = 0.0;
      for (int kb = 0; kb < nkbA + nkbC; ++kb) {
        if (kb < nkd) {
          ok = mbar_wait(&full[stage], phase, abort, p.status);
          __syncwarp();
          if (__any_sync(0xffffffffu, !ok)) {
            ok = false;
            break;
          }
          const uint8_t* a_row = smem + stage * stage_bytes + rl * 128;
          float f = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 q = *reinterpret_cast<const uint4*>(a_row + (((half_id * 4 + c) ^ (rl & 7)) << 4));
            const bf16* e = reinterpret_cast<const bf16*>(&q);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float v = __bfloat162float(e[j]);
              f = fmaf(v, v, f);
            }
          }
          ss += (double)f;
          __syncwarp();
          if (lane == 0) mbar_arrive(&rmsd[stage]);
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      rms_part[half_id * 128 + rl] = (float)ss;
      __syncwarp();
      if (lane == 0) mbar_arrive(rmsx);
      ok = mbar_wait(rmsx, it & 1, abort, p.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !ok)) break;
      const float rr =
          (float)(1.0 / sqrt(((double)rms_part[rl] + (double)rms_part[128 + rl]) / p.d + (double)p.eps));
      if (half_id == 0 && valid && rank == 0) p.r[row] = rr;
      // phase B: h = r * acc as hi | mid | lo bf16 parts.  The ring is idle until every part is
      // stored (phase A's loads are consumed, and the producer waits for hxr before phase C), so
      // box (chunk j, part) is staged at ring offset (3 j + part) * 16 KB and the storer issues
      // all the TMA stores at once.
      ok = mbar_wait(tfullA, it & 1, abort, p.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !ok)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(wq * 32) << 16);
#pragma unroll 1
      for (int j = 0; j < lh / 64; ++j) {
        uint32_t v[32];
        tmem_ld32(tbase + j * 64 + half_id * 32, v);
        tc_wait_ld();
        float a[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) a[q] = __uint_as_float(v[q]) * rr;
#pragma unroll
        for (int part = 0; part < 3; ++part) {
          uint32_t w[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const bf16 h0 = __float2bfloat16_rn(a[2 * q]), h1 = __float2bfloat16_rn(a[2 * q + 1]);
            __nv_bfloat162 ph = __halves2bfloat162(h0, h1);
            w[q] = *reinterpret_cast<uint32_t*>(&ph);
            a[2 * q] -= __bfloat162float(h0);
            a[2 * q + 1] -= __bfloat162float(h1);
          }
          uint8_t* box = smem + (3 * j + part) * 16384;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(box + sw128_offset(rl, half_id * 4 + q)) =
                make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(tempA);
        mbar_arrive(hxs);
      }
      if (storer) {
        ok = mbar_wait(hxs, it & 1, abort, p.status);
        __syncwarp();
        if (__any_sync(0xffffffffu, !ok)) break;
        if (lane == 0) {
          for (int j = 0; j < lh / 64; ++j)
            for (int part = 0; part < 3; ++part)
              tma_store_2d(&p.tm_hx, smem + (3 * j + part) * 16384, part * p.l + (int)rank * lh + j * 64, row0);
          bulk_commit();
          bulk_wait_all();  // the h parts are in global memory (and the ring is free) before phase C
          mbar_arrive(hxr);  // own barrier first: the peer's next arrival comes after it
          if (ns == 2) mbar_arrive_cluster(mapa_shared(smem_u32(hxr), rank ^ 1u));
        }
        __syncwarp();
      }
      // phase D: s = sigmoid(z + c), fp32, 32 columns per box (16 per warp).  On this CTA's last
      // tile the ring is idle once phase C's products are done (no loads follow), so every box is
      // staged there (box j at j * 16 KB) and stored at once; otherwise the two-box ring of emit.
      ok = mbar_wait(tfullC, it & 1, abort, p.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !ok)) break;
      tc_fence_after();
      const bool last_tile = tile + stride >= num_tiles;
      bool nan = false;
      uint32_t w[16];
#pragma unroll 1
      for (int j = 0; ok && j < eh / 32; ++j) {
        uint32_t v[16], vs[16];
        tmem_ld16(tbase + lh + j * 32 + half_id * 16, v);
        if (dual) tmem_ld16(tbase + j * 32 + half_id * 16, vs);
        float cj = c_lane[0];  // select by unrolled compares: no dynamic register indexing
#pragma unroll
        for (int jj = 1; jj < 8; ++jj)
          if (jj == j) cj = c_lane[jj];
        tc_wait_ld();
        if (dual) {
#pragma unroll
          for (int q = 0; q < 16; ++q) v[q] = __float_as_uint(__uint_as_float(v[q]) + __uint_as_float(vs[q]));
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          // lane m of the warp holds offset j*32 + m (loaded at the start of the kernel)
          const float cb = __shfl_sync(0xffffffffu, cj, half_id * 16 + q);
          const float o = sigmoidf_acc(__uint_as_float(v[q]) + cb);
          nan |= (o != o);
          w[q] = __float_as_uint(o);
        }
        if (last_tile) {
          uint8_t* box = smem + j * 16384;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(box + sw128_offset(rl, half_id * 4 + q)) =
                make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        } else {
          ok = emit(w, &p.tm_s, (int)rank * eh + j * 32, row0);
        }
      }
      if (!ok) break;
      if (last_tile) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(sds);
        if (storer) {
          ok = mbar_wait(sds, 0, abort, p.status);
          __syncwarp();
          if (__any_sync(0xffffffffu, !ok)) break;
          if (lane == 0) {
            for (int j = 0; j < eh / 32; ++j) tma_store_2d(&p.tm_s, smem + j * 16384, (int)rank * eh + j * 32, row0);
            bulk_commit();
          }
          __syncwarp();
        }
      }
      if (nan && valid) set_status(p.status, LMOE_STATUS_NAN_SCORE);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempC);
    }
    if (storer && lane == 0) bulk_wait_all();
  }

  __syncthreads();
  if (ns == 2) cluster_sync_all();  // no remote arrival is still on its way to this CTA
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

}  // namespace lmoe
