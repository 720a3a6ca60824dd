// Block-scaled 8-bit routed-expert GEMMs (MXFP8) for sm_100a: tcgen05.mma.kind::mxf8f6f4 with
// per-32-element power-of-two scales held in tensor memory.
//
// Format (the reading the oracle's lowp module fixes): E4M3 elements, rounded to nearest with
// ties to even and saturated at 448; one scale 2^X per 32 consecutive elements along K, with
// X = floor(log2 max|v|) - 8 clamped to [-127, 127] (-127 for an all-zero block), stored as the
// UE8M0 byte X + 127.  The MMA multiplies the elements exactly, scales each 32-element block's
// products by its two operands' scales and accumulates in fp32 (one instruction of shape
// 128 x N x 32 per scale block).
//
// Scale layout.  The scales of a 128-row tile and a 128-element K-block (4 blocks of 32) form a
// 512-byte atom: byte 16 i + 4 j + b is the scale of row i + 32 j, 32-element block b
// (i < 32, j < 4, b < 4).  In global memory the atoms of a matrix are stored tile-major, then by
// K-block: atom (t, kb) at byte ((t * nkb) + kb) * 512.  A tcgen05.cp of shape 32x128b.warpx4
// copies an atom into four TMEM columns of all four lane quarters (lane 32 q + i, column j, byte
// b), where the MMA reads the scale of row m from column m / 32, lane m % 32 and byte sf_id.
//
// Grouped like the engine's bf16 grouped mode: M-tiles of 128 gathered token rows (every expert's
// rows start on a multiple of 128; an expert's last tile loads only its valid rows, rounded up to
// 32), N-tiles of 128 weight rows, K-blocks of 128 elements (one 128-byte swizzle atom, four MMAs).
// CTA = 10 warps: warp 0 issues TMA loads of the two operand tiles and bulk copies of their two
// scale atoms into a 6-stage ring, warp 1 copies each stage's atoms into TMEM (two buffers,
// alternating by K-block, at 32-column-aligned addresses) and issues the four MMAs that read
// them, warps 2-9 drain the other accumulator.
//  Q8_SWIGLU (gate/up, N columns interleaved in groups of 64 gate + 64 linear): act = silu(g) * u
//    for 32 features per thread, quantised to MXFP8 right there (the thread holds exactly one
//    32-element block of its row) and stored as 32 element bytes and one scale byte (atom layout).
//  Q8_BF16 (down): out bf16.
// Every wait is bounded as in the engine.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace lmoe {

enum Q8Epilogue : int { Q8_SWIGLU = 0, Q8_BF16 = 1 };

struct Q8Params {
  CUtensorMap tmA;          // A elements [rows, K] u8, box 128 x 128
  CUtensorMap tmA_part[3];  // the same with boxes of 32, 64, 96 rows
  CUtensorMap tmB;          // B elements [groups * b_rows, K] u8, box 128 x 128
  const uint8_t* a_sf;      // A scale atoms (rows / 128 tiles x K / 128 blocks x 512 bytes)
  const uint8_t* b_sf;      // B scale atoms
  const int2* mtile_table;  // (expert | valid rows << 16, first row)
  const int* num_mtiles;
  int n_tiles;              // N / 128
  int b_rows;               // B rows per expert
  int nkb;                  // K / 128 (at most 32)
  uint8_t* out_q;           // Q8_SWIGLU: act elements [rows, N / 2]
  uint8_t* out_sf;          //            act scale atoms (K-blocks of N / 2)
  bf16* out_bf;             // Q8_BF16: [rows, N]
  int n_out;                // output columns of the whole GEMM (N, or N / 2 for SwiGLU)
  uint32_t* status;
};

constexpr int kQ8Stages = 6;
constexpr int kQ8StageBytes = 32768 + 1024;  // A tile, B tile, A scale atom, B scale atom
constexpr int kQ8BarOffset = kQ8Stages * kQ8StageBytes;
constexpr int kQ8SmemBytes = kQ8BarOffset + 256 + 1024;
constexpr int kQ8Threads = kTcThreads;

// Byte offset of the scale of row r, 32-element block c (of K) in a matrix's atom layout with nkb
// K-blocks of 128.
__host__ __device__ __forceinline__ long long mx_atom_offset(long long r, int c, int nkb) {
  return ((r >> 7) * nkb + (c >> 2)) * 512 + 16 * (r & 31) + 4 * ((r & 127) >> 5) + (c & 3);
}

// MXFP8 scale exponent of a block whose largest magnitude is amax: floor(log2 amax) - 8, clamped
// to [-127, 127]; -127 for a zero block (or one below fp32's normal range).
__device__ __forceinline__ int mx_scale_exp(float amax) {
  if (!(amax > 0.f)) return -127;
  const int e = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127;  // floor(log2) of a normal number
  if (e == -127) return -127;                                     // subnormal: X would be below -127
  const int X = e - 8;
  return X < -127 ? -127 : (X > 127 ? 127 : X);
}

// 2^-X as an fp32 number (X in [-127, 119], so the result is a normal number).
__device__ __forceinline__ float pow2_neg(int X) { return __uint_as_float((uint32_t)(127 - X) << 23); }

// Four scaled values as E4M3 bytes (round to nearest even, saturating at 448), first in the low byte.
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// Quantises 32 values (one block) to MXFP8: eight words of element bytes and the scale byte.
__device__ __forceinline__ uint32_t mx_quant32(const float (&v)[32], uint32_t (&q)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int X = mx_scale_exp(amax);
  const float s = pow2_neg(X);
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = e4m3x4(v[4 * i] * s, v[4 * i + 1] * s, v[4 * i + 2] * s, v[4 * i + 3] * s);
  return (uint32_t)(X + 127);
}

// Instruction descriptor, kind::mxf8f6f4: D fp32, A and B E4M3, both K-major, UE8M0 scales,
// M = 128, N = n; sf_id selects the byte of each scale word the MMA reads.
__device__ __forceinline__ uint32_t idesc_mxf8(int n, int a_sf_id, int b_sf_id) {
  return ((uint32_t)b_sf_id << 4) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | ((uint32_t)(128 >> 4) << 24) |
         ((uint32_t)a_sf_id << 29);
}

__device__ __forceinline__ void tc_mma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate));
}

// Shared-memory descriptor of a 32-row x 16-byte matrix stored row after row, without swizzle:
// core matrices of 8 rows x 16 bytes, 128 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_rows16(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128u >> 4) << 16;
  d |= (uint64_t)(128u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  return d;
}
// Copies a 512-byte scale atom from shared memory into TMEM columns [taddr, taddr + 4) of all four
// lane quarters (ordered with this thread's later MMAs).
__device__ __forceinline__ void tc_cp_atom(uint32_t taddr, uint32_t saddr) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(smem_desc_rows16(saddr)));
}
// Bulk copy (no tensor map) of `bytes` from global to shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

template <int EPI>
__global__ void __launch_bounds__(kQ8Threads, 1) q8_gemm_kernel(const __grid_constant__ Q8Params p) {
  constexpr int S = kQ8Stages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQ8BarOffset);
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
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
    for (int i = 0; i < 3; ++i) tma_prefetch_desc(&p.tmA_part[i]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // TMEM columns: accumulators [0, 256); scale buffer i (by K-block parity): A at 256 + 64 i,
  // B at 288 + 64 i (four columns each, at 32-column-aligned addresses)
  const uint32_t sf_base = tmem_base + 256;
  pdl_wait();
  pdl_trigger();
  const int num_tiles = *p.num_mtiles * p.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int mt = tile / p.n_tiles, nt = tile - mt * p.n_tiles;
        const int2 e_r = p.mtile_table[mt];
        const int q = ((e_r.x >> 16) + 31) >> 5;
        const int row0 = e_r.y, brow0 = (e_r.x & 0xFFFF) * p.b_rows + nt * 128;
        const CUtensorMap* amap = q < 4 ? &p.tmA_part[q - 1] : &p.tmA;
        for (int kb = 0; kb < p.nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = smem + stage * kQ8StageBytes;
          mbar_expect_tx(&full[stage], (uint32_t)(q * 32 * 128 + 16384 + 1024));
          tma_load_2d(a_dst, amap, &full[stage], kb * 128, row0);
          // no L2 evict-first hint on the weights: an expert's slice serves row tiles that run at
          // about the same time (the hint made the wide layer's 8-bit experts slower)
          tma_load_2d(a_dst + 16384, &p.tmB, &full[stage], kb * 128, brow0);
          bulk_load(a_dst + 32768, p.a_sf + ((size_t)(row0 >> 7) * p.nkb + kb) * 512, 512, &full[stage]);
          bulk_load(a_dst + 32768 + 512, p.b_sf + ((size_t)(brow0 >> 7) * p.nkb + kb) * 512, 512, &full[stage]);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok)
        for (int i = 0; i < S; ++i)
          if ((armed >> i) & 1u) mbar_drain(&full[i], (armed_parity >> i) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t par = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], par ^ 1u, abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 128;
        for (int kb = 0; kb < p.nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * kQ8StageBytes);
          const uint32_t b_addr = a_addr + 16384;
          // this K-block's scale atoms into the scale buffer of its parity, then its four MMAs
          const uint32_t sfa = sf_base + (kb & 1) * 64, sfb = sfa + 32;
          tc_cp_atom(sfa, a_addr + 32768);
          tc_cp_atom(sfb, a_addr + 32768 + 512);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_mxf8(d_tmem, smem_desc_sw128(a_addr + k * 32), smem_desc_sw128(b_addr + k * 32),
                        idesc_mxf8(128, k, k), sfa, sfb, (kb | k) != 0);
          tc_commit(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      if (!ok) {
        tc_commit(drain);
        mbar_drain(drain, 0);
      }
    }
  } else {
    // ---------------- epilogue warps 2..9: TMEM lane quarter (warp % 4), column half (warp - 2) / 4
    const int wq = warp & 3;
    const int half_id = (warp - 2) >> 2;
    const int rl = wq * 32 + lane;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
      const int mt = tile / p.n_tiles, nt = tile - mt * p.n_tiles;
      const int row = p.mtile_table[mt].y + rl;
      const int acc = it & 1;
      ok = mbar_wait(&tfull[acc], (it >> 1) & 1, abort, p.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(wq * 32) << 16) + acc * 128;
      if constexpr (EPI == Q8_SWIGLU) {
        // gate columns [32 half, +32), linear columns 64 further: act features nt * 64 + 32 half + [0, 32)
        uint32_t gv[32], uv[32];
        tmem_ld32(tbase + half_id * 32, gv);
        tmem_ld32(tbase + 64 + half_id * 32, uv);
        tc_wait_ld();
        float a[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = silu_fast(__uint_as_float(gv[i])) * __uint_as_float(uv[i]);
        uint32_t qw[8];
        const uint32_t sfb = mx_quant32(a, qw);
        const int col = nt * 64 + half_id * 32;
        uint4* dst = reinterpret_cast<uint4*>(p.out_q + (size_t)row * p.n_out + col);
        dst[0] = make_uint4(qw[0], qw[1], qw[2], qw[3]);
        dst[1] = make_uint4(qw[4], qw[5], qw[6], qw[7]);
        p.out_sf[mx_atom_offset(row, col >> 5, p.n_out >> 7)] = (uint8_t)sfb;
      } else {
        // columns [64 half, +64) of this N-tile, bf16
#pragma unroll 1
        for (int j = 0; j < 2; ++j) {
          uint32_t v[32];
          tmem_ld32(tbase + half_id * 64 + j * 32, v);
          tc_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          uint4* dst = reinterpret_cast<uint4*>(p.out_bf + (size_t)row * p.n_out + nt * 128 + half_id * 64 + j * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
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
    tmem_dealloc(tmem_base, 512);
  }
}

// --------------------------------------------------------------------------- quantisation kernels
// MXFP8 of rows of a matrix along its columns (the GEMM's K): one thread per 32-element block.
// Source: bf16 [rows, cols] (parts == 1), or the hi | mid | lo bf16 parts of fp32 values
// ([rows, 3 cols], parts == 3), summed back to fp32 first.  out: [rows, cols] elements; scale
// bytes row after row ([rows, cols / 32], atom == 0) or in the atom layout (atom == 1).
__global__ void __launch_bounds__(256) mx_quant_rows_kernel(const bf16* __restrict__ src, int parts, long long rows,
                                                            int cols, uint8_t* __restrict__ out,
                                                            uint8_t* __restrict__ out_sf, int atom) {
  pdl_wait();
  pdl_trigger();
  const int nb = cols / 32;
  const long long n = rows * nb;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / nb;
    const int b = (int)(i - r * nb);
    float v[32];
    const bf16* s = src + r * (long long)cols * parts + b * 32;
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      const uint4 h = *reinterpret_cast<const uint4*>(s + j);
      const bf16* he = reinterpret_cast<const bf16*>(&h);
#pragma unroll
      for (int t = 0; t < 8; ++t) v[j + t] = __bfloat162float(he[t]);
    }
    if (parts == 3) {
#pragma unroll
      for (int part = 1; part < 3; ++part) {
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          const uint4 h = *reinterpret_cast<const uint4*>(s + part * cols + j);
          const bf16* he = reinterpret_cast<const bf16*>(&h);
#pragma unroll
          for (int t = 0; t < 8; ++t) v[j + t] += __bfloat162float(he[t]);
        }
      }
    }
    uint32_t q[8];
    const uint32_t sf = mx_quant32(v, q);
    uint4* d = reinterpret_cast<uint4*>(out + r * cols + b * 32);
    d[0] = make_uint4(q[0], q[1], q[2], q[3]);
    d[1] = make_uint4(q[4], q[5], q[6], q[7]);
    out_sf[atom ? mx_atom_offset(r, b, cols / 128) : r * nb + b] = (uint8_t)sf;
  }
}

// MXFP8 of the routed experts' gate and linear projections, rows interleaved in groups of 64 as
// the SwiGLU epilogue reads them (out row (j / 64) 128 + j % 64 = w1[j], 64 further = w3[j], per
// expert), along l, scales in the atom layout; one thread per 32-element block.
__global__ void __launch_bounds__(256) mx_quant_w13_kernel(const bf16* __restrict__ w1, const bf16* __restrict__ w3,
                                                           int E, int h, int l, uint8_t* __restrict__ out,
                                                           uint8_t* __restrict__ out_sf) {
  const int nb = l / 32;
  const long long n = (long long)E * 2 * h * nb;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long orow = i / nb;
    const int b = (int)(i - orow * nb);
    const int e = (int)(orow / (2 * h)), r = (int)(orow - (long long)e * 2 * h);
    const int within = r & 127, j = (r >> 7) * 64 + (within & 63);
    const bf16* s = (within < 64 ? w1 : w3) + ((long long)e * h + j) * l + b * 32;
    float v[32];
#pragma unroll
    for (int q = 0; q < 32; q += 8) {
      const uint4 hv = *reinterpret_cast<const uint4*>(s + q);
      const bf16* he = reinterpret_cast<const bf16*>(&hv);
#pragma unroll
      for (int t = 0; t < 8; ++t) v[q + t] = __bfloat162float(he[t]);
    }
    uint32_t qw[8];
    const uint32_t sf = mx_quant32(v, qw);
    uint4* d = reinterpret_cast<uint4*>(out + orow * l + b * 32);
    d[0] = make_uint4(qw[0], qw[1], qw[2], qw[3]);
    d[1] = make_uint4(qw[4], qw[5], qw[6], qw[7]);
    out_sf[mx_atom_offset(orow, b, l / 128)] = (uint8_t)sf;
  }
}

// Copies each (token, slot) pair's MXFP8 row (cols elements, cols / 32 scale bytes stored row
// after row) into row prow[pair] of the padded expert layout, its scales into the atom layout;
// one warp per pair.
__global__ void __launch_bounds__(256) gather_q8_kernel(const uint8_t* __restrict__ src, const uint8_t* __restrict__ src_sf,
                                                        int cols, const int* __restrict__ prow, int npairs, int k,
                                                        uint8_t* __restrict__ dst, uint8_t* __restrict__ dst_sf) {
  pdl_wait();
  pdl_trigger();
  const int pair = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (pair >= npairs) return;
  const int t = pair / k, r = prow[pair];
  const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)t * cols);
  uint4* d = reinterpret_cast<uint4*>(dst + (size_t)r * cols);
  for (int v = lane; v < cols / 16; v += 32) d[v] = s[v];
  const uint8_t* ss = src_sf + (size_t)t * (cols / 32);
  for (int c = lane; c < cols / 32; c += 32) dst_sf[mx_atom_offset(r, c, cols / 128)] = ss[c];
}

}  // namespace lmoe
