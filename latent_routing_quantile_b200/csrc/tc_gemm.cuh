// Persistent tcgen05 GEMM for sm_100a: C[M, N] = A[M, K] * B[N, K]^T, A and B bf16 K-major,
// fp32 accumulation in tensor memory (TMEM), with the layer's epilogues fused.
//
// CTA = 10 warps: warp 0 issues TMA loads into a STAGES-deep shared-memory ring, warp 1 issues
// tcgen05.mma (one thread) into one of two TMEM accumulators, warps 2-9 drain the other
// accumulator (tcgen05.ld) through the epilogue while the next tile is multiplied.  Two
// epilogue warps share each TMEM lane quarter and split its columns, so the element-wise
// epilogue math keeps pace with the tensor core.  Tiles are
// 128 x BN, K steps of 64 (one 128-byte swizzle atom).  The grid is at most one CTA per SM and
// walks the tile list with a stride of gridDim.x.
//
// Grouped mode (routed experts): M-tiles come from a device table of (expert, first row) built
// after the routing counts, B rows are offset by expert * b_rows_per_group, and rows past the
// expert's segment end are computed but never stored.
//
// K is described by up to 6 segments, each naming which A tensor map and which A and B columns
// its k-blocks read; this expresses concatenated-K products ([z | a_s] [W_up | Ws2]^T) and the
// split-precision router (hi/mid/lo products) without copying operands.
#pragma once

#include "common.cuh"

namespace lmoe {

enum TcEpilogue : int {
  EPI_F32 = 0,     // out fp32 = acc
  EPI_BF16 = 1,    // out bf16 = acc
  EPI_SWIGLU = 2,  // columns interleaved in groups of 64 (gate, linear): out bf16 = silu(g)*u,
                   // both scaled by row_scale[row] first when row_scale != null
  EPI_DOWN3 = 3,   // v = row_scale[row]*acc; out bf16 [.., 3*split]: hi, mid, lo parts of v
  EPI_ROUTER = 4,  // out fp32 = sigmoid(acc + col_bias[col])
};

struct KSeg {
  int a_map;  // 0 or 1
  int a_col;  // first A column of the segment
  int b_col;  // first B column of the segment
  int nkb;    // k-blocks of 64
};

struct TcParams {
  CUtensorMap tmA[2];
  CUtensorMap tmB;
  KSeg seg[6];
  int nseg;
  int grouped;
  int M;                      // rows (non-grouped)
  int n_tiles;                // N / BN
  const int2* mtile_table;    // grouped: (expert, first row)
  const int* num_mtiles;      // grouped: number of table entries (device)
  const int* seg_off;         // grouped: expert row offsets [E+1]
  int b_rows_per_group;       // grouped: B rows per expert
  void* out;
  int ldo;                    // output row pitch in elements
  int split;                  // EPI_DOWN3: width of each of the three parts
  const float* row_scale;
  const float* col_bias;
  uint32_t* status;
};

template <int BN>
struct TcCfg {
  static constexpr int kABytes = 128 * 128;              // 128 rows x 64 bf16
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (192 * 1024) / kStageBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // barriers + alignment slack
};

struct TileInfo {
  int row0, row_end, b_row0, n0;
};

__device__ __forceinline__ TileInfo tc_tile(const TcParams& p, int tile, int BN) {
  TileInfo ti;
  int mt = tile / p.n_tiles, nt = tile - mt * p.n_tiles;
  ti.n0 = nt * BN;
  if (p.grouped) {
    int2 e_r = p.mtile_table[mt];
    ti.row0 = e_r.y;
    ti.row_end = p.seg_off[e_r.x + 1];
    ti.b_row0 = e_r.x * p.b_rows_per_group + ti.n0;
  } else {
    ti.row0 = mt * 128;
    ti.row_end = p.M;
    ti.b_row0 = ti.n0;
  }
  return ti;
}

__device__ __forceinline__ int tc_num_tiles(const TcParams& p) {
  int mt = p.grouped ? *p.num_mtiles : (p.M + 127) / 128;
  return mt * p.n_tiles;
}

constexpr int kEpiWarps = 8;
constexpr int kTcThreads = 64 + 32 * kEpiWarps;

template <int BN, int EPI>
__global__ void __launch_bounds__(kTcThreads, 1) tc_gemm_kernel(const __grid_constant__ TcParams p) {
  using C = TcCfg<BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tmA[0]);
    tma_prefetch_desc(&p.tmA[1]);
    tma_prefetch_desc(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = tc_num_tiles(p);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // per-stage bits, for the abort drain
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        TileInfo ti = tc_tile(p, tile, BN);
        for (int s = 0; ok && s < p.nseg; ++s) {
          const KSeg sg = p.seg[s];
          for (int kb = 0; kb < sg.nkb; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort, p.status)) {
              ok = false;
              break;
            }
            uint8_t* a_dst = smem + stage * C::kStageBytes;
            uint8_t* b_dst = a_dst + C::kABytes;
            mbar_expect_tx(&full[stage], C::kStageBytes);
            tma_load_2d(a_dst, &p.tmA[sg.a_map], &full[stage], sg.a_col + kb * 64, ti.row0);
            tma_load_2d(b_dst, &p.tmB, &full[stage], sg.b_col + kb * 64, ti.b_row0);
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      if (!ok) {
        // let every load this thread issued land before the CTA's shared memory is released
        for (int i = 0; i < S; ++i)
          if ((armed >> i) & 1u) mbar_drain(&full[i], (armed_parity >> i) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        int kbi = 0;
        for (int s = 0; ok && s < p.nseg; ++s) {
          const int nkb = p.seg[s].nkb;
          for (int kb = 0; kb < nkb; ++kb, ++kbi) {
            if (!mbar_wait(&full[stage], phase, abort, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + stage * C::kStageBytes);
            const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              tc_mma_bf16(d_tmem, smem_desc_sw128(a_addr + k * 32), smem_desc_sw128(b_addr + k * 32),
                          idesc, (kbi | k) != 0);
            }
            tc_commit(&empty[stage]);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      if (!ok) {
        // wait (bounded) for the MMAs already issued before TMEM is released
        tc_commit(drain);
        mbar_drain(drain, 0);
      }
    }
  } else {
    // ---------------- epilogue warps 2..9: TMEM lane quarter (warp % 4), column half (warp-2)/4
    const int wq = warp & 3;
    const int half_id = (warp - 2) >> 2;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      bool ok = mbar_wait(&tfull[acc], acc_phase, abort, p.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !ok)) break;
      tc_fence_after();
      TileInfo ti = tc_tile(p, tile, BN);
      const int row = ti.row0 + wq * 32 + lane;
      const bool valid = row < ti.row_end;
      const uint32_t tbase = tmem_base + ((uint32_t)(wq * 32) << 16) + acc * BN;
      const float rs = (p.row_scale != nullptr && valid) ? p.row_scale[row] : 1.0f;

      if constexpr (EPI == EPI_SWIGLU) {
        // item i = (group g = i / 2, part = i % 2): gate columns g*128 + part*32 .. +31, linear
        // columns 64 further; items alternate between the two warps of a lane quarter
#pragma unroll 1
        for (int item = half_id; item < BN / 64; item += 2) {
          const int g = item >> 1, part = item & 1;
          uint32_t gv[32], uv[32];
          tmem_ld32(tbase + g * 128 + part * 32, gv);
          tmem_ld32(tbase + g * 128 + 64 + part * 32, uv);
          tc_wait_ld();
          if (valid) {
            bf16* o = reinterpret_cast<bf16*>(p.out) + (size_t)row * p.ldo + (ti.n0 >> 1) + g * 64 + part * 32;
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float g0 = __uint_as_float(gv[2 * j]) * rs, g1 = __uint_as_float(gv[2 * j + 1]) * rs;
              const float u0 = __uint_as_float(uv[2 * j]) * rs, u1 = __uint_as_float(uv[2 * j + 1]) * rs;
              pk[j] = pack_bf16x2(silu_fast(g0) * u0, silu_fast(g1) * u1);
            }
            uint4* o4 = reinterpret_cast<uint4*>(o);
#pragma unroll
            for (int j = 0; j < 4; ++j) o4[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = half_id; c < BN / 32; c += 2) {
          uint32_t v[32];
          tmem_ld32(tbase + c * 32, v);
          tc_wait_ld();
          if (!valid) continue;
          const int col = ti.n0 + c * 32;
          if constexpr (EPI == EPI_F32) {
            float4* o4 = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (size_t)row * p.ldo + col);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              o4[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                  __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          } else if constexpr (EPI == EPI_BF16) {
            uint4* o4 = reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(p.out) + (size_t)row * p.ldo + col);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              o4[j] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1])),
                                 pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                                 pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                                 pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
          } else if constexpr (EPI == EPI_DOWN3) {
            // v = r * acc, stored as hi + mid + lo bf16 parts (exact to fp32's 24 bits)
            bf16* base = reinterpret_cast<bf16*>(p.out) + (size_t)row * p.ldo + col;
            uint32_t hi[16], mid[16], lo[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float a0 = __uint_as_float(v[2 * j]) * rs, a1 = __uint_as_float(v[2 * j + 1]) * rs;
              const bf16 h0 = __float2bfloat16_rn(a0), h1 = __float2bfloat16_rn(a1);
              const float r0 = a0 - __bfloat162float(h0), r1 = a1 - __bfloat162float(h1);
              const bf16 m0 = __float2bfloat16_rn(r0), m1 = __float2bfloat16_rn(r1);
              const float q0 = r0 - __bfloat162float(m0), q1 = r1 - __bfloat162float(m1);
              __nv_bfloat162 ph = __halves2bfloat162(h0, h1), pm = __halves2bfloat162(m0, m1);
              hi[j] = *reinterpret_cast<uint32_t*>(&ph);
              mid[j] = *reinterpret_cast<uint32_t*>(&pm);
              lo[j] = pack_bf16x2(q0, q1);
            }
            uint4* oh = reinterpret_cast<uint4*>(base);
            uint4* om = reinterpret_cast<uint4*>(base + p.split);
            uint4* ol = reinterpret_cast<uint4*>(base + 2 * p.split);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              oh[j] = make_uint4(hi[4 * j], hi[4 * j + 1], hi[4 * j + 2], hi[4 * j + 3]);
              om[j] = make_uint4(mid[4 * j], mid[4 * j + 1], mid[4 * j + 2], mid[4 * j + 3]);
              ol[j] = make_uint4(lo[4 * j], lo[4 * j + 1], lo[4 * j + 2], lo[4 * j + 3]);
            }
          } else if constexpr (EPI == EPI_ROUTER) {
            float4* o4 = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (size_t)row * p.ldo + col);
            const float4* cb4 = reinterpret_cast<const float4*>(p.col_bias + col);
            bool nan = false;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 cb = cb4[j];
              float4 o;
              o.x = sigmoidf_acc(__uint_as_float(v[4 * j]) + cb.x);
              o.y = sigmoidf_acc(__uint_as_float(v[4 * j + 1]) + cb.y);
              o.z = sigmoidf_acc(__uint_as_float(v[4 * j + 2]) + cb.z);
              o.w = sigmoidf_acc(__uint_as_float(v[4 * j + 3]) + cb.w);
              nan |= (o.x != o.x) | (o.y != o.y) | (o.z != o.z) | (o.w != o.w);
              o4[j] = o;
            }
            if (nan) set_status(p.status, LMOE_STATUS_NAN_SCORE);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace lmoe
