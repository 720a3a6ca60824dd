// Persistent tcgen05 GEMM for sm_100a: C[M, N] = A[M, K] * B[N, K]^T, A and B bf16 K-major,
// fp32 accumulation in tensor memory (TMEM), with the layer's epilogues fused.
//
// CTA = 10 warps: warp 0 issues TMA loads into a STAGES-deep shared-memory ring, warp 1 issues
// tcgen05.mma (one thread) into one of two TMEM accumulators, warps 2-9 drain the other
// accumulator (tcgen05.ld) through the epilogue while the next tile is multiplied.  Two
// epilogue warps share each TMEM lane quarter and split its columns, so the element-wise
// epilogue math keeps pace with the tensor core.  Results leave through shared memory: each
// step the epilogue warps fill one 16 KB box (128 rows x 128 bytes, 128-byte swizzle) of a
// two-box staging ring and warp 2 issues a TMA tensor store of it, so global writes are whole
// lines instead of one 16-byte piece per row per thread.  Tiles are
// 128 x BN, K steps of 64 (one 128-byte swizzle atom).  The grid is at most one CTA per SM and
// walks the tile list with a stride of gridDim.x.
//
// Grouped mode (routed experts): M-tiles come from a device table of (expert, valid rows, first
// row) built after the routing counts, and B rows are offset by expert * b_rows_per_group.
// Every expert's rows start on a multiple of 128, so a tile never holds rows of two experts.
// With `trim`, a tile with R < 128 valid rows loads and stores only ceil(R/32)*32 rows (tensor
// maps with 32/64/96-row boxes): the padding rows cost no memory traffic.  The MMA still runs
// 128 rows; rows past the load hold stale shared memory, and only their own output rows, which
// are never stored, depend on them.
//
// K is described by up to 12 segments, each naming which A tensor map and which A and B columns
// its k-blocks read; this expresses concatenated-K products ([z | a_s] [W_up | Ws2]^T) without
// copying operands, and the split-precision products of the fp32 layer: an fp32 operand is held
// as three bf16 parts [hi | mid | lo] along K (hi + mid + lo = the value to fp32's 24 bits) and
// A B^T is the sum of the six significant part products (lo lo, mid lo and lo mid fall below
// fp32's rounding), one segment each, all accumulated in fp32 in TMEM.
//
// EPI_ROUTER (the split-precision router, not paired) reads three segments, the hi, mid and lo
// parts of h and of the router weights, chunk by chunk: the three stages of a 64-column chunk
// (part q of A and of B in stage q) feed all six significant products, five small ones
// ((mid,mid) (lo,hi) (hi,lo) (mid,hi) (hi,mid)) into one accumulator and (hi,hi) into a second,
// so each part is loaded once and the small terms are summed among themselves; the epilogue adds
// the two.  Its accumulators take 2 BN TMEM columns each (BN <= 128).
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
  EPI_SWIGLU3 = 5, // as EPI_SWIGLU with an accurate SiLU, the fp32 result stored as hi, mid, lo bf16
                   // parts (columns part * split + c) for the next split-precision product
  EPI_F32_DEEP = 7,    // as EPI_F32 with four output staging boxes (for streams of fp32 results:
                       // the experts' weight gradients)
  EPI_SWIGLU_BWD = 6,  // acc = dL/d act of a SwiGLU; with its pre-activations p1 (gate) and p3
                       // (linear) read from aux, out bf16: dL/dp1 = acc p3 silu'(p1) at column c and
                       // dL/dp3 = acc silu(p1) at column split + c; rows past the tile's valid rows 0
};

struct KSeg {
  int a_map;  // 0 or 1
  int a_col;  // first A column of the segment (MN-major A: first K row)
  int b_col;  // first B column of the segment (MN-major B: first K row)
  int nkb;    // k-blocks of 64
  int b_map;  // 0: tmB, 1 / 2: tmB2[0] / tmB2[1]
};

struct TcParams {
  CUtensorMap tmA[2];
  CUtensorMap tmB;
  CUtensorMap tmOut;          // output: box 64 x 128 (bf16) or 32 x 128 (fp32), 128-byte swizzle
  CUtensorMap tmA_part[3];    // trim: tmA[0] with boxes of 32, 64, 96 rows
  CUtensorMap tmOut_part[3];  // trim: tmOut with boxes of 32, 64, 96 rows
  KSeg seg[12];
  int nseg;
  int grouped;
  int M;                      // rows (non-grouped)
  int n_tiles;                // N / BN
  const int2* mtile_table;    // grouped: (expert, first row)
  const int* num_mtiles;      // grouped: number of table entries (device)
  int b_rows_per_group;       // grouped: B rows per expert
  int M_rows;                 // rows whose row_scale may be read (non-grouped: M)
  int split;                  // EPI_DOWN3: column offset between the three parts
  const float* row_scale;
  const float* col_bias;
  int trim;                   // grouped: move only the valid rows of a tile, rounded up to 32
  int hint_a, hint_b;         // 1: load A / B with L2 evict_first (read once, not again soon)
  int hint_out;               // 1: store the output with L2 evict_last (the next kernel reads it)
  int band_n;                 // non-grouped: N-tiles per band of the tile order (0: row-major order)
  uint32_t* status;
  // ---- the layer backward's products
  CUtensorMap tmB2[2];        // B maps of segments with b_map 1 and 2
  CUtensorMap tmOut2;         // output of the rows at or past out_split (re-based to row 0)
  int out_split;              // 0: one output map
  int a_mn, b_mn;             // operand stored MN-major: A as [K, M], B as [K, N] (64 x 64 boxes)
  int grouped_k;              // expert weight gradients: K runs over one expert's rows
  int k_groups;               // grouped_k: experts (tiles = k_groups x M-tiles x N-tiles)
  const int* k_first;         // grouped_k: first row of each expert, unpadded ...
  const int* k_pad;           // ... plus this: its first row in the padded layout
  const int* k_rows;          // grouped_k: rows of each expert
  const bf16* aux;            // EPI_SWIGLU_BWD: [rows, 2 split] pre-activations, gate and linear
  int ld_aux;                 // columns interleaved in groups of 64 (as the forward's weights)
  int out_pre;                // EPI_SWIGLU: also store the bf16 pre-activations (the accumulator
                              // scaled by row_scale, gate and linear columns as accumulated) to
                              // tmOut2, for a backward pass (no trim)
  int k_split;                // > 1 (non-grouped, one segment, EPI_F32): the k-blocks are cut into
                              // k_split ranges, one tile each, whose results are added into the
                              // output (zeroed first) by TMA reductions
};

// PAIR = 1: a cluster of two CTAs computes one 256 x BN tile with tcgen05.mma.cta_group::2; each
// CTA holds 128 rows of A and BN/2 rows of B per stage.
// EXTRA: shared memory the epilogue keeps for itself, taken from the load ring.
template <int BN, int PAIR = 0, int EXTRA = 0>
struct TcCfg {
  static constexpr int kABytes = 128 * 128;              // 128 rows x 64 bf16
  static constexpr int kBBytes = (PAIR ? BN / 2 : BN) * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (192 * 1024 - EXTRA) / kStageBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kOutOffset = kStages * kStageBytes;    // two 16 KB output boxes
  static constexpr int kAuxOffset = kOutOffset + 2 * 16384;   // the epilogue's own (EXTRA bytes)
  static constexpr int kBarOffset = kAuxOffset + EXTRA;
  static constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // barriers + alignment slack
};

// EPI_SWIGLU_BWD stages the pre-activations each epilogue warp reads: per warp, gate and linear
// values of its 32 rows x 32 columns, rows 80 bytes apart (64 bytes of data + 16 of padding, so
// that eight lanes reading eight rows hit distinct banks).
constexpr int kAuxWarpBytes = 2 * 32 * 80;
// Output staging boxes of an epilogue (boxes past two live in its EXTRA bytes).  Four cost a stage
// of the load ring; they pay only where the output stream is what limits a kernel.
__host__ __device__ constexpr int tc_out_boxes(int epi) { return epi == EPI_F32_DEEP ? 4 : 2; }
__host__ __device__ constexpr int tc_epi_extra(int epi) {
  return epi == EPI_SWIGLU_BWD ? 8 * kAuxWarpBytes : (tc_out_boxes(epi) - 2) * 16384;
}
template <int BN, int EPI, int PAIR>
using TcCfgFor = TcCfg<BN, PAIR, tc_epi_extra(EPI)>;

struct TileInfo {
  int row0, b_row0, n0;
  int q;         // 32-row quarters of the tile that are loaded and stored (4 = all)
  int out_y;     // first output row of the tile
  int sel;       // output map: 0 tmOut (or its trimmed forms), 1 tmOut2
  int valid;     // rows of the tile that hold data (grouped: the expert's rows; else up to M)
  int ak0, bk0;  // first K row of an MN-major A / B operand (grouped modes: the expert's)
  int kb0, nkb;  // grouped_k / k_split: first k-block and k-blocks of the tile; nkb -1: the
                 // segments' own counts
};

// Tile order: row-major over (M-tile, N-tile), or, with band_n > 0 (non-grouped), band by band:
// all M-tiles of N-tiles [b band_n, (b+1) band_n) before the next band, so the tiles that run at
// the same time share a band of B that stays in L2 instead of streaming all of B per M-tile.
// GEN: the general modes (split K, grouped K, a second output map) exist; the forward's products
// are compiled without them.
template <bool GEN>
__device__ __forceinline__ TileInfo tc_tile(const TcParams& p, int tile, int BN, int pair, uint32_t rank) {
  TileInfo ti;
  int mt, nt;
  ti.q = 4;
  ti.sel = 0;
  ti.valid = 128;
  ti.ak0 = 0;
  ti.bk0 = 0;
  ti.kb0 = 0;
  ti.nkb = -1;
  if (GEN && p.k_split > 1) {
    // split s of a one-segment K: tiles [s*base, (s+1)*base) cover k-blocks [s*nkb/S, (s+1)*nkb/S)
    const int base = (pair ? (p.M + 255) >> 8 : (p.M + 127) >> 7) * p.n_tiles;
    const int sp = tile / base;
    tile -= sp * base;
    const int nk = p.seg[0].nkb;
    ti.kb0 = (int)(((long long)sp * nk) / p.k_split);
    ti.nkb = (int)(((long long)(sp + 1) * nk) / p.k_split) - ti.kb0;
  }
  if (GEN && p.grouped_k) {
    // expert-major: all (M-tile, N-tile) pairs of one expert's gradient, then the next expert's
    const int per = ((p.M + 127) >> 7) * p.n_tiles;
    const int e = tile / per;
    const int idx = tile - e * per;
    mt = idx / p.n_tiles;
    nt = idx - mt * p.n_tiles;
    ti.n0 = nt * BN;
    ti.row0 = mt * 128;
    ti.b_row0 = ti.n0;
    ti.ak0 = ti.bk0 = p.k_first[e] + p.k_pad[e];
    ti.nkb = (p.k_rows[e] + 63) >> 6;
    int m = ti.row0;
    if (p.out_split && m >= p.out_split) {
      ti.sel = 1;
      m -= p.out_split;
    }
    ti.out_y = e * (p.out_split ? p.out_split : p.M) + m;
    return ti;
  }
  if (p.band_n > 0 && !p.grouped) {
    const int m_tiles = pair ? (p.M + 255) / 256 : (p.M + 127) / 128;
    const int per_band = m_tiles * p.band_n;
    const int band = tile / per_band;
    const int idx = tile - band * per_band;
    const int nb = min(p.band_n, p.n_tiles - band * p.band_n);  // the last band may be narrower
    mt = idx / nb;
    nt = band * p.band_n + (idx - mt * nb);
  } else {
    mt = tile / p.n_tiles;
    nt = tile - mt * p.n_tiles;
  }
  ti.n0 = nt * BN;
  if (pair) {  // 256-row tiles; this CTA owns rows 128*rank.. and B rows BN/2*rank..
    ti.row0 = mt * 256 + (int)rank * 128;
    ti.b_row0 = ti.n0 + (int)rank * (BN / 2);
    ti.valid = min(128, p.M - ti.row0);  // may be 0 or less: no row of this CTA holds data
  } else if (p.grouped) {
    int2 e_r = p.mtile_table[mt];
    ti.row0 = e_r.y;
    ti.b_row0 = (e_r.x & 0xFFFF) * p.b_rows_per_group + ti.n0;
    ti.bk0 = (e_r.x & 0xFFFF) * p.b_rows_per_group;
    ti.valid = e_r.x >> 16;
    if (p.trim) ti.q = ((e_r.x >> 16) + 31) >> 5;
  } else {
    ti.row0 = mt * 128;
    ti.b_row0 = ti.n0;
    ti.valid = min(128, p.M - ti.row0);
  }
  ti.out_y = ti.row0;
  if (GEN && p.out_split && ti.row0 >= p.out_split) {
    ti.sel = 1;
    ti.out_y -= p.out_split;
  }
  return ti;
}

template <bool GEN>
__device__ __forceinline__ int tc_num_tiles(const TcParams& p, int pair) {
  if (GEN && p.grouped_k) return p.k_groups * ((p.M + 127) >> 7) * p.n_tiles;
  if (GEN && p.k_split > 1) return p.k_split * (pair ? (p.M + 255) >> 8 : (p.M + 127) >> 7) * p.n_tiles;
  int mt = p.grouped ? *p.num_mtiles : (pair ? (p.M + 255) / 256 : (p.M + 127) / 128);
  return mt * p.n_tiles;
}

constexpr int kEpiWarps = 8;
constexpr int kTcThreads = 64 + 32 * kEpiWarps;

// GEN = 0: without the backward's modes (MN-major operands, per-segment B maps, grouped or split
// K, a second output map), whose runtime branches in the producer, MMA and epilogue loops cost the
// forward's products 3-7% at the replica's width; the host picks the form from the parameters.
template <int BN, int EPI, int PAIR, int GEN>
__global__ void __launch_bounds__(kTcThreads, 1) tc_gemm_kernel(const __grid_constant__ TcParams p) {
  constexpr bool G = GEN != 0;
  using C = TcCfgFor<BN, EPI, PAIR>;
  constexpr int S = C::kStages;
  constexpr int NB = tc_out_boxes(EPI);  // output staging boxes (the ones past two in the EXTRA bytes)
  constexpr bool kSplit3 = EPI == EPI_ROUTER && !PAIR;  // chunk-major split-precision products
  constexpr int kAccCols = kSplit3 ? 2 * BN : BN;       // TMEM columns of one accumulator buffer
  constexpr uint32_t kTmemCols = 2 * kAccCols;
  static_assert(kTmemCols <= 512 && (!kSplit3 || S >= 3), "router tiles are at most 128 wide");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* bfull = tempty + 2;   // output box written by all epilogue warps
  uint64_t* bfree = bfull + NB;   // output box read by its TMA store
  uint64_t* drain = bfree + NB;
  uint8_t* obox = smem + C::kOutOffset;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0 = the pair's MMA issuer
  const bool leader = rank == 0;
  // pairs walk the tile list together: pair index and count
  const int first = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int stride = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], PAIR ? 2 * kEpiWarps : kEpiWarps);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(&bfull[i], kEpiWarps);
      mbar_init(&bfree[i], 1);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tmA[0]);
    tma_prefetch_desc(&p.tmA[1]);
    tma_prefetch_desc(&p.tmB);
    tma_prefetch_desc(&p.tmOut);
    if (p.trim)
      for (int i = 0; i < 3; ++i) {
        tma_prefetch_desc(&p.tmA_part[i]);
        tma_prefetch_desc(&p.tmOut_part[i]);
      }
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // the peer's barriers exist before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // operands, tile table and row scales come from earlier kernels
  pdl_trigger();
  const int num_tiles = tc_num_tiles<G>(p, PAIR);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // per-stage bits, for the abort drain
      const uint64_t pol_first = l2_evict_first();
      bool ok = true;
      // the tile after this one is looked up one tile ahead: in grouped mode that is a global load
      // whose latency would otherwise stall the issue of every tile's first loads
      TileInfo ti_next = tc_tile<G>(p, first < num_tiles ? first : 0, BN, PAIR, rank);
      for (int tile = first; ok && tile < num_tiles; tile += stride) {
        const TileInfo ti = ti_next;
        if (tile + stride < num_tiles) ti_next = tc_tile<G>(p, tile + stride, BN, PAIR, rank);
        // k-blocks segment by segment, or (split router) chunk by chunk over the three segments
        const int nouter = kSplit3 ? p.seg[0].nkb : p.nseg;
        for (int o = 0; ok && o < nouter; ++o) {
          const int ninner = kSplit3 ? 3 : ((G && ti.nkb >= 0) ? ti.nkb : p.seg[o].nkb);
          for (int in = 0; in < ninner; ++in) {
            const KSeg sg = p.seg[kSplit3 ? in : o];
            const int kb = kSplit3 ? o : (G ? ti.kb0 + in : in);
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort, p.status)) {
              ok = false;
              break;
            }
            uint8_t* a_dst = smem + stage * C::kStageBytes;
            uint8_t* b_dst = a_dst + C::kABytes;
            if constexpr (PAIR) {
              // both CTAs' bytes complete the leader's full barrier; the leader expects all of them
              const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
              if (leader) mbar_expect_tx(&full[stage], 2 * C::kStageBytes);
              const CUtensorMap* bmap = (G && sg.b_map) ? &p.tmB2[sg.b_map - 1] : &p.tmB;
              if (G && p.a_mn) {  // this CTA's 128 rows of M as two 64 x 64 boxes
                const int ky = ti.ak0 + sg.a_col + kb * 64;
                tma_load_2d_pair(a_dst, &p.tmA[sg.a_map], bar0, ti.row0, ky);
                tma_load_2d_pair(a_dst + 8192, &p.tmA[sg.a_map], bar0, ti.row0 + 64, ky);
              } else {
                tma_load_2d_pair(a_dst, &p.tmA[sg.a_map], bar0, sg.a_col + kb * 64, ti.row0);
              }
              if (G && p.b_mn) {  // this CTA's BN/2 columns of N, 64 at a time
                const int ky = ti.bk0 + sg.b_col + kb * 64;
#pragma unroll
                for (int c = 0; c < BN / 128; ++c) tma_load_2d_pair(b_dst + c * 8192, bmap, bar0, ti.b_row0 + 64 * c, ky);
              } else {
                tma_load_2d_pair(b_dst, bmap, bar0, sg.b_col + kb * 64, ti.b_row0);
              }
            } else if (G && (p.a_mn | p.b_mn)) {
              // MN-major operands: one 64 x 64 box per 64 columns of M (N), 64 K rows each
              const CUtensorMap* bmap = (G && sg.b_map) ? &p.tmB2[sg.b_map - 1] : &p.tmB;
              mbar_expect_tx(&full[stage], (uint32_t)(C::kABytes + C::kBBytes));
              if (p.a_mn) {
                const int ky = ti.ak0 + sg.a_col + kb * 64;
                tma_load_2d(a_dst, &p.tmA[sg.a_map], &full[stage], ti.row0, ky);
                tma_load_2d(a_dst + 8192, &p.tmA[sg.a_map], &full[stage], ti.row0 + 64, ky);
              } else {
                tma_load_2d(a_dst, &p.tmA[sg.a_map], &full[stage], sg.a_col + kb * 64, ti.row0);
              }
              if (p.b_mn) {
                const int ky = ti.bk0 + sg.b_col + kb * 64;
#pragma unroll
                for (int c = 0; c < BN / 64; ++c) tma_load_2d(b_dst + c * 8192, bmap, &full[stage], ti.n0 + 64 * c, ky);
              } else {
                tma_load_2d(b_dst, bmap, &full[stage], sg.b_col + kb * 64, ti.b_row0);
              }
            } else {
              const CUtensorMap* amap = ti.q < 4 ? &p.tmA_part[ti.q - 1] : &p.tmA[sg.a_map];
              const CUtensorMap* bmap = (G && sg.b_map) ? &p.tmB2[sg.b_map - 1] : &p.tmB;
              mbar_expect_tx(&full[stage], (uint32_t)(ti.q * 32 * 128 + C::kBBytes));
              if (p.hint_a)
                tma_load_2d_hint(a_dst, amap, &full[stage], sg.a_col + kb * 64, ti.row0, pol_first);
              else
                tma_load_2d(a_dst, amap, &full[stage], sg.a_col + kb * 64, ti.row0);
              if (p.hint_b)
                tma_load_2d_hint(b_dst, bmap, &full[stage], sg.b_col + kb * 64, ti.b_row0, pol_first);
              else
                tma_load_2d(b_dst, bmap, &full[stage], sg.b_col + kb * 64, ti.b_row0);
            }
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      if (!ok && leader) {
        // let every load issued land before shared memory is released (for a pair, the leader's
        // barriers count both CTAs' loads, and the final cluster barrier holds the peer)
        for (int i = 0; i < S; ++i)
          if ((armed >> i) & 1u) mbar_drain(&full[i], (armed_parity >> i) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (the even CTA of a pair issues for both)
      constexpr uint32_t idesc = idesc_bf16_f32(BN, PAIR ? 256 : 128);
      // MN-major operands: transpose bits of the instruction descriptor
      const uint32_t idesc_t = G ? idesc | (p.a_mn ? 1u << 15 : 0u) | (p.b_mn ? 1u << 16 : 0u) : idesc;
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = first; ok && tile < num_tiles; tile += stride, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        if constexpr (kSplit3) {
          // per chunk: stage q holds part q (hi, mid, lo) of A and of B; small products into the
          // accumulator's first BN columns, smallest first, (hi, hi) into the second BN
          constexpr uint32_t kPa = 1u | (2u << 2) | (0u << 4) | (1u << 6) | (0u << 8);
          constexpr uint32_t kPb = 1u | (0u << 2) | (2u << 4) | (0u << 6) | (1u << 8);
          const int nch = p.seg[0].nkb;
          for (int kk = 0; ok && kk < nch; ++kk) {
            uint32_t a_addr[3], b_addr[3];
            int st3[3];
#pragma unroll
            for (int q = 0; q < 3; ++q) {
              if (!mbar_wait(&full[stage], phase, abort, p.status)) {
                ok = false;
                break;
              }
              a_addr[q] = smem_u32(smem + stage * C::kStageBytes);
              b_addr[q] = a_addr[q] + C::kABytes;
              st3[q] = stage;
              if (++stage == S) {
                stage = 0;
                phase ^= 1u;
              }
            }
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int pr = 0; pr < 5; ++pr) {
              const int pa = (int)((kPa >> (2 * pr)) & 3u), pb = (int)((kPb >> (2 * pr)) & 3u);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                tc_mma_bf16(d_tmem, smem_desc_sw128(a_addr[pa] + k * 32), smem_desc_sw128(b_addr[pb] + k * 32), idesc,
                            (kk | pr | k) != 0);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_bf16(d_tmem + BN, smem_desc_sw128(a_addr[0] + k * 32), smem_desc_sw128(b_addr[0] + k * 32), idesc,
                          (kk | k) != 0);
#pragma unroll
            for (int q = 0; q < 3; ++q) tc_commit(&empty[st3[q]]);
          }
          if (ok) tc_commit(&tfull[acc]);
          continue;
        }
        int kbi = 0;
        const int tnkb = (G && (p.grouped_k || p.k_split > 1)) ? tc_tile<G>(p, tile, BN, PAIR, rank).nkb : -1;
        for (int s = 0; ok && s < p.nseg; ++s) {
          const int nkb = tnkb >= 0 ? tnkb : p.seg[s].nkb;
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
              // K-major: the next 16 K columns are 32 bytes on in each 128-byte row; MN-major: 16
              // K rows of 128 bytes further
              const uint64_t ad = (G && p.a_mn) ? smem_desc_mn128(a_addr + k * 2048) : smem_desc_sw128(a_addr + k * 32);
              const uint64_t bd = (G && p.b_mn) ? smem_desc_mn128(b_addr + k * 2048) : smem_desc_sw128(b_addr + k * 32);
              if constexpr (PAIR)
                tc_mma_bf16_pair(d_tmem, ad, bd, idesc_t, (kbi | k) != 0);
              else
                tc_mma_bf16(d_tmem, ad, bd, idesc_t, (kbi | k) != 0);
            }
            if constexpr (PAIR)
              tc_commit_pair(&empty[stage]);
            else
              tc_commit(&empty[stage]);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (ok) {
          if constexpr (PAIR)
            tc_commit_pair(&tfull[acc]);
          else
            tc_commit(&tfull[acc]);
        }
      }
      if (!ok) {
        // wait (bounded) for the MMAs already issued before TMEM is released
        if constexpr (PAIR)
          tc_commit_pair(drain);
        else
          tc_commit(drain);
        mbar_drain(drain, 0);
      }
    }
  } else {
    // ---------------- epilogue warps 2..9: TMEM lane quarter (warp % 4), column half (warp-2)/4
    const int wq = warp & 3;
    const int half_id = (warp - 2) >> 2;
    const int rl = wq * 32 + lane;          // row of the tile this thread owns
    const bool storer = (warp == 2);        // warp 2 issues the TMA stores
    int it = 0;
    uint32_t step = 0;                      // output boxes so far (alternating staging buffers)
    bool ok = true;
    // Writes this thread's 64 bytes into the current box, then (storer) stores the box.
    const CUtensorMap* omap = &p.tmOut;  // this tile's output map (trim: only its valid rows)
    auto emit = [&](const uint32_t (&w)[16], int x, int y, const CUtensorMap* to = nullptr) -> bool {
      const int buf = (int)(step % NB);
      const uint32_t par = (step / NB) & 1u;
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
          if (to)
            tma_store_2d(to, box, x, y);
          else if (G && p.k_split > 1)
            tma_reduce_add_2d(omap, box, x, y);
          else if (p.hint_out)
            tma_store_2d_hint(omap, box, x, y, l2_evict_last());
          else
            tma_store_2d(omap, box, x, y);
          bulk_commit();
          if (step >= NB - 1) {
            bulk_wait_read<NB - 1>();  // the box stored NB - 1 steps ago has been read: it is free
            mbar_arrive(&bfree[(step - (NB - 1)) % NB]);
          }
        }
        __syncwarp();
      }
      ++step;
      return true;
    };
    uint4 pf[8];           // EPI_SWIGLU_BWD: pre-activations fetched ahead
    bool pf_next = false;  // EPI_SWIGLU_BWD: pf holds the next tile's first step
    for (int tile = first; ok && tile < num_tiles; tile += stride, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      float c_lane[BN / 32];  // router column offsets of this tile, one per lane and step
      if constexpr (EPI == EPI_ROUTER) {
        const int n0 = tc_tile<G>(p, tile, BN, PAIR, rank).n0;
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) c_lane[j] = p.col_bias[n0 + j * 32 + lane];
      } else {
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) c_lane[j] = 0.f;
      }
      // tile table entry and row scale are loaded before the wait, so their latency overlaps it
      const TileInfo ti = tc_tile<G>(p, tile, BN, PAIR, rank);
      const int row = ti.row0 + rl;
      const float rs = (p.row_scale != nullptr && row < p.M_rows) ? p.row_scale[row] : 1.0f;
      ok = mbar_wait(&tfull[acc], acc_phase, abort, p.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      omap = (G && ti.sel) ? &p.tmOut2 : (ti.q < 4 ? &p.tmOut_part[ti.q - 1] : &p.tmOut);
      const bool zero_acc = G && ti.nkb == 0;  // grouped_k: an expert without rows has a zero gradient
      const uint32_t tbase = tmem_base + ((uint32_t)(wq * 32) << 16) + acc * kAccCols;
      uint32_t w[16];

      if constexpr (EPI == EPI_SWIGLU) {
        // step j: output columns n0/2 + j*64 .. +63; this warp's 32 of them come from gate
        // columns j*128 + half*32 and linear columns 64 further
#pragma unroll 1
        for (int j = 0; ok && j < BN / 128; ++j) {
          uint32_t gv[32], uv[32];
          tmem_ld32(tbase + j * 128 + half_id * 32, gv);
          tmem_ld32(tbase + j * 128 + 64 + half_id * 32, uv);
          tc_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float g0 = __uint_as_float(gv[2 * q]) * rs, g1 = __uint_as_float(gv[2 * q + 1]) * rs;
            const float u0 = __uint_as_float(uv[2 * q]) * rs, u1 = __uint_as_float(uv[2 * q + 1]) * rs;
            w[q] = pack_bf16x2(silu_fast(g0) * u0, silu_fast(g1) * u1);
          }
          ok = emit(w, (ti.n0 >> 1) + j * 64, ti.out_y);
          if (p.out_pre) {
            // the pre-activations, in the accumulator's own column order
#pragma unroll
            for (int q = 0; q < 16; ++q)
              w[q] = pack_bf16x2(__uint_as_float(gv[2 * q]) * rs, __uint_as_float(gv[2 * q + 1]) * rs);
            if (ok) ok = emit(w, ti.n0 + j * 128, ti.out_y, &p.tmOut2);
#pragma unroll
            for (int q = 0; q < 16; ++q)
              w[q] = pack_bf16x2(__uint_as_float(uv[2 * q]) * rs, __uint_as_float(uv[2 * q + 1]) * rs);
            if (ok) ok = emit(w, ti.n0 + j * 128 + 64, ti.out_y, &p.tmOut2);
          }
        }
      } else if constexpr (EPI == EPI_SWIGLU3) {
#pragma unroll 1
        for (int j = 0; ok && j < BN / 128; ++j) {
          uint32_t gv[32], uv[32];
          tmem_ld32(tbase + j * 128 + half_id * 32, gv);
          tmem_ld32(tbase + j * 128 + 64 + half_id * 32, uv);
          tc_wait_ld();
          float a[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) a[q] = siluf(__uint_as_float(gv[q]) * rs) * (__uint_as_float(uv[q]) * rs);
#pragma unroll 1
          for (int part = 0; ok && part < 3; ++part) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const bf16 h0 = __float2bfloat16_rn(a[2 * q]), h1 = __float2bfloat16_rn(a[2 * q + 1]);
              __nv_bfloat162 ph = __halves2bfloat162(h0, h1);
              w[q] = *reinterpret_cast<uint32_t*>(&ph);
              a[2 * q] -= __bfloat162float(h0);  // remainder for the next part
              a[2 * q + 1] -= __bfloat162float(h1);
            }
            ok = emit(w, part * p.split + (ti.n0 >> 1) + j * 64, ti.out_y);
          }
        }
      } else if constexpr (EPI == EPI_BF16) {
#pragma unroll 1
        for (int j = 0; ok && j < BN / 64; ++j) {
          uint32_t v[32];
          tmem_ld32(tbase + j * 64 + half_id * 32, v);
          tc_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q)
            w[q] = pack_bf16x2(__uint_as_float(v[2 * q]) * rs, __uint_as_float(v[2 * q + 1]) * rs);
          ok = emit(w, ti.n0 + j * 64, ti.out_y);
        }
      } else if constexpr (EPI == EPI_SWIGLU_BWD) {
        // step j: accumulator columns c = n0 + j*64 + half*32 + q hold dL/d act; the gate and linear
        // pre-activations of column c sit at aux columns (c/64)*128 + c%64 and 64 further.  Each
        // warp copies the 32 x 32 gate and linear values of its rows and columns with whole
        // 64-byte row pieces (8 rows per load instruction) into its staging rows, one step ahead,
        // then every lane reads its own row from there.
        const bool live = rl < ti.valid;
        uint8_t* stg = smem + C::kAuxOffset + (warp - 2) * kAuxWarpBytes;
        // copies step j of tile t's pre-activations for this warp's 32 rows and columns into pf
        auto fetch = [&](const TileInfo& t, int j) {
          const int c0 = t.n0 + j * 64 + half_id * 32;
          const int g0 = ((c0 >> 6) << 7) + (c0 & 63);
          const int rbase = t.row0 + wq * 32;
          const int nlive = t.valid - wq * 32;  // rows of this warp's quarter that hold data
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = lane + 32 * i, which = c >> 7, rr = (c >> 2) & 31, cc = c & 3;
            pf[i] = rr < nlive ? ldg_nc_v4(p.aux + (size_t)(rbase + rr) * p.ld_aux + g0 + which * 64 + cc * 8)
                               : make_uint4(0, 0, 0, 0);
          }
        };
        if (!pf_next) fetch(ti, 0);  // else the previous tile's last step fetched it
#pragma unroll 1
        for (int j = 0; ok && j < BN / 64; ++j) {
          uint32_t v[32];
          tmem_ld32(tbase + j * 64 + half_id * 32, v);
          const int c0 = ti.n0 + j * 64 + half_id * 32;
          __syncwarp();  // every lane has read the previous step's staging rows
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = lane + 32 * i, which = c >> 7, rr = (c >> 2) & 31, cc = c & 3;
            *reinterpret_cast<uint4*>(stg + which * (kAuxWarpBytes / 2) + rr * 80 + cc * 16) = pf[i];
          }
          __syncwarp();
          // the next step's values, or the next tile's first step's, load while this step computes
          if (j + 1 < BN / 64) {
            fetch(ti, j + 1);
          } else {
            pf_next = tile + stride < num_tiles;
            if (pf_next) fetch(tc_tile<G>(p, tile + stride, BN, PAIR, rank), 0);
          }
          uint4 pg[4], pu[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            pg[i] = *reinterpret_cast<const uint4*>(stg + lane * 80 + i * 16);
            pu[i] = *reinterpret_cast<const uint4*>(stg + kAuxWarpBytes / 2 + lane * 80 + i * 16);
          }
          tc_wait_ld();
          uint32_t w3[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const uint32_t gw = (&pg[q >> 2].x)[q & 3], uw = (&pu[q >> 2].x)[q & 3];
            float d1[2], d3[2];
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
              const float g = __uint_as_float(hlf ? (gw & 0xFFFF0000u) : (gw << 16));
              const float u = __uint_as_float(hlf ? (uw & 0xFFFF0000u) : (uw << 16));
              const float sg = sigmoidf_acc(g);
              const float as = __uint_as_float(v[2 * q + hlf]) * sg;  // dL/dact * sigmoid(g)
              d1[hlf] = live ? as * u * fmaf(g, 1.0f - sg, 1.0f) : 0.0f;
              d3[hlf] = live ? as * g : 0.0f;
            }
            w[q] = pack_bf16x2(d1[0], d1[1]);
            w3[q] = pack_bf16x2(d3[0], d3[1]);
          }
          ok = emit(w, c0 - half_id * 32, ti.out_y);
          if (ok) ok = emit(w3, p.split + c0 - half_id * 32, ti.out_y);
        }
      } else if constexpr (EPI == EPI_DOWN3) {
        // v = r * acc, stored as hi + mid + lo bf16 parts (exact to fp32's 24 bits), one box each
#pragma unroll 1
        for (int j = 0; ok && j < BN / 64; ++j) {
          uint32_t v[32];
          tmem_ld32(tbase + j * 64 + half_id * 32, v);
          tc_wait_ld();
          float a[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) a[q] = __uint_as_float(v[q]) * rs;
#pragma unroll 1
          for (int part = 0; ok && part < 3; ++part) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const bf16 h0 = __float2bfloat16_rn(a[2 * q]), h1 = __float2bfloat16_rn(a[2 * q + 1]);
              __nv_bfloat162 ph = __halves2bfloat162(h0, h1);
              w[q] = *reinterpret_cast<uint32_t*>(&ph);
              a[2 * q] -= __bfloat162float(h0);   // remainder for the next part
              a[2 * q + 1] -= __bfloat162float(h1);
            }
            ok = emit(w, part * p.split + ti.n0 + j * 64, ti.out_y);
          }
        }
      } else {
        // EPI_F32 / EPI_ROUTER: step j = 32 fp32 columns, 16 per warp.  The router's column offsets
        // of this tile sit one per lane (lane m: offset n0 + j*32 + m), loaded before the waits.
        bool nan = false;
#pragma unroll 1
        for (int j = 0; ok && j < BN / 32; ++j) {
          uint32_t v[16], vs[16];
          if constexpr (kSplit3) {
            tmem_ld16(tbase + BN + j * 32 + half_id * 16, v);  // (hi, hi)
            tmem_ld16(tbase + j * 32 + half_id * 16, vs);      // the five small products
          } else if (zero_acc) {
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = 0u;
          } else {
            tmem_ld16(tbase + j * 32 + half_id * 16, v);
          }
          float cj = c_lane[0];
#pragma unroll
          for (int jj = 1; jj < BN / 32; ++jj)
            if (jj == j) cj = c_lane[jj];
          tc_wait_ld();
          if constexpr (kSplit3) {
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = __float_as_uint(__uint_as_float(v[q]) + __uint_as_float(vs[q]));
          }
          if constexpr (EPI == EPI_ROUTER) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float o = sigmoidf_acc(__uint_as_float(v[q]) + __shfl_sync(0xffffffffu, cj, half_id * 16 + q));
              nan |= (o != o);
              w[q] = __float_as_uint(o);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) w[q] = v[q];
          }
          ok = emit(w, ti.n0 + j * 32, ti.out_y);
        }
        if (nan && row < p.M_rows) set_status(p.status, LMOE_STATUS_NAN_SCORE);
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR)
          mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));  // the leader's barrier
        else
          mbar_arrive(&tempty[acc]);
      }
    }
    if (storer && lane == 0) bulk_wait_all();  // every store has left shared memory and landed
  }

  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // both CTAs are done with TMEM and each other's barriers
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, kTmemCols);
    else
      tmem_dealloc(tmem_base, kTmemCols);
  }
  if constexpr (PAIR) cluster_sync_all();
}

}  // namespace lmoe
