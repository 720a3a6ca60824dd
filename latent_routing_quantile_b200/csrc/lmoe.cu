// Host side of the C ABI declared in include/lmoe.h: validation, weight repacking, workspace,
// tensor maps, and the launch sequence of one forward.  Nothing here synchronises inside a
// forward; every launch goes to the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "common.cuh"
#include "route.cuh"
#include "bwd.cuh"
#include "tc_gemm.cuh"
#include "k1_router.cuh"
#include "q8_gemm.cuh"

using namespace lmoe;

namespace {

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tensor map of a row-major matrix with a 128-byte swizzle (the layout the MMA descriptors and the
// staged epilogue expect).
bool make_map_t(CUtensorMap* m, const void* base, long long rows, long long cols, long long pitch, int box_rows,
                bool f32) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const long long es_bytes = f32 ? 4 : 2;
  if (((uintptr_t)base & 15) || ((pitch * es_bytes) & 15) || rows <= 0 || cols <= 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(pitch * es_bytes)};
  cuuint32_t box[2] = {f32 ? 32u : 64u, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
             dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// bf16 matrix [rows, cols], row pitch `pitch` elements; box = 64 columns (128 bytes) x box_rows.
bool make_map(CUtensorMap* m, const void* base, long long rows, long long cols, long long pitch, int box_rows) {
  return make_map_t(m, base, rows, cols, pitch, box_rows, false);
}
// 8-bit matrix [rows, cols]; box = 128 columns (128 bytes) x box_rows, 128-byte swizzle.
bool make_map_u8(CUtensorMap* m, const void* base, long long rows, long long cols, long long pitch, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  if (((uintptr_t)base & 15) || (pitch & 15) || rows <= 0 || cols <= 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)pitch};
  cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// fp32 matrix; box = 32 columns (128 bytes) x box_rows.
bool make_map_f32(CUtensorMap* m, const void* base, long long rows, long long cols, long long pitch, int box_rows) {
  return make_map_t(m, base, rows, cols, pitch, box_rows, true);
}

int pick_bn(int n) { return n % 256 == 0 ? 256 : (n % 128 == 0 ? 128 : 64); }

// N-tiles per band of a non-grouped GEMM's tile order (tc_tile): B's band (bn columns x K bf16
// elements per N-tile) at most 32 MB, so that it and the A rows of the tiles running beside it
// stay in the 126 MB L2; 0 (row-major order) when all of B fits.
int pick_band(int n_tiles, int bn, long long k_elems) {
  const long long per_tile = (long long)bn * k_elems * 2;
  const long long fit = (32ll << 20) / per_tile;
  return fit >= n_tiles ? 0 : (int)std::max(1ll, fit);
}

// Tile width for a non-grouped GEMM of M rows and N columns: the widest that divides N and still
// gives every SM a tile (min_bn = 128 for the SwiGLU epilogue, whose column groups are 128 wide).
int pick_bn_for(long long M, int N, int sms, int min_bn) {
  const long long mt = (M + 127) / 128;
  for (int bn = 256; bn >= min_bn; bn >>= 1)
    if (N % bn == 0 && mt * (N / bn) >= sms) return bn;
  for (int bn = min_bn; bn <= 256; bn <<= 1)
    if (N % bn == 0) return bn;
  return min_bn;
}

// Raises a kernel's dynamic shared-memory limit once per device; `done` is the caller's own
// per-kernel flag word (one bit per device).
template <typename K>
cudaError_t ensure_smem_attr(K kern, int bytes, unsigned& done) {
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned bit = 1u << (dev & 31);
  if (done & bit) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done |= bit;
  return e;
}

// Launches `kern` with programmatic stream serialisation, so its blocks may be scheduled while
// the previous kernel of the stream drains (every kernel of the layer calls pdl_wait() before
// touching data another kernel writes), and for cluster_x > 1 in clusters of cluster_x CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                     Args... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  memset(attr, 0, sizeof(attr));
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Whether a launch uses the engine's general modes (MN-major operands, per-segment B maps,
// grouped or split K, a second output map): only the backward's products do, and they run the
// kernel compiled with them; the forward's products run the one without.
bool tc_general(const TcParams& p) {
  if (p.a_mn || p.b_mn || p.grouped_k || p.k_split > 1 || p.out_split) return true;
  for (int s = 0; s < p.nseg; ++s)
    if (p.seg[s].b_map) return true;
  return false;
}

// Forms an epilogue is compiled in: 0 without the general modes, 1 with them, 2 both.
constexpr int tc_forms(int epi) {
  return (epi == EPI_BF16 || epi == EPI_F32) ? 2 : ((epi == EPI_SWIGLU_BWD || epi == EPI_F32_DEEP) ? 1 : 0);
}

template <int BN, int EPI, int PAIR, int GEN>
cudaError_t launch_tc_g(const TcParams& p, int grid, cudaStream_t st) {
  auto kern = tc_gemm_kernel<BN, EPI, PAIR, GEN>;
  static unsigned done = 0;
  constexpr int smem = TcCfgFor<BN, EPI, PAIR>::kSmemBytes;
  cudaError_t e = ensure_smem_attr(kern, smem, done);
  if (e != cudaSuccess) return e;
  // pairs: clusters of 2 along x, grid even
  return launch_k(kern, dim3(PAIR ? (unsigned)(grid & ~1) : (unsigned)grid), dim3(kTcThreads), smem, st,
                  PAIR ? 2 : 1, p);
}

// The form the parameters need; a general launch of an epilogue compiled only without the general
// modes is refused.
template <int BN, int EPI, int PAIR>
cudaError_t launch_tc_f(const TcParams& p, int grid, cudaStream_t st) {
  constexpr int f = tc_forms(EPI);
  const bool gen = tc_general(p);
  if constexpr (f == 2) {
    return gen ? launch_tc_g<BN, EPI, PAIR, 1>(p, grid, st) : launch_tc_g<BN, EPI, PAIR, 0>(p, grid, st);
  } else if constexpr (f == 1) {
    return launch_tc_g<BN, EPI, PAIR, 1>(p, grid, st);
  } else {
    if (gen) return cudaErrorInvalidValue;
    return launch_tc_g<BN, EPI, PAIR, 0>(p, grid, st);
  }
}

template <int BN, int EPI>
cudaError_t launch_tc_t(const TcParams& p, int grid, cudaStream_t st) {
  return launch_tc_f<BN, EPI, 0>(p, grid, st);
}

// Two-CTA (cta_group::2) variant: clusters of 2 along x, grid even.
template <int BN, int EPI>
cudaError_t launch_tc_pair_t(const TcParams& p, int grid, cudaStream_t st) {
  return launch_tc_f<BN, EPI, 1>(p, grid, st);
}

template <int EPI>
cudaError_t launch_tc_e(const TcParams& p, int bn, int grid, cudaStream_t st) {
  switch (bn) {
    case 256:
      if constexpr (EPI == EPI_ROUTER) return cudaErrorInvalidValue;  // two accumulators: BN <= 128
      else return launch_tc_t<256, EPI>(p, grid, st);
    case 128: return launch_tc_t<128, EPI>(p, grid, st);
    default:
      if constexpr (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU3) return cudaErrorInvalidValue;
      else return launch_tc_t<64, EPI>(p, grid, st);
  }
}

cudaError_t launch_tc(const TcParams& p, int epi, int bn, int grid, cudaStream_t st) {
  switch (epi) {
    case EPI_F32: return launch_tc_e<EPI_F32>(p, bn, grid, st);
    case EPI_BF16: return launch_tc_e<EPI_BF16>(p, bn, grid, st);
    case EPI_SWIGLU: return launch_tc_e<EPI_SWIGLU>(p, bn, grid, st);
    case EPI_DOWN3: return launch_tc_e<EPI_DOWN3>(p, bn, grid, st);
    case EPI_SWIGLU3: return launch_tc_e<EPI_SWIGLU3>(p, bn, grid, st);
    case EPI_SWIGLU_BWD: return launch_tc_e<EPI_SWIGLU_BWD>(p, bn, grid, st);
    case EPI_F32_DEEP: return launch_tc_e<EPI_F32_DEEP>(p, bn, grid, st);
    default: return launch_tc_e<EPI_ROUTER>(p, bn, grid, st);
  }
}

// Pair launches exist for tile widths 128 and 256 and the bf16 / SwiGLU / fp32 / SwiGLU-backward /
// three-part epilogues.
cudaError_t launch_tc_pair(const TcParams& p, int epi, int bn, int grid, cudaStream_t st) {
  if (epi == EPI_SWIGLU) return bn == 256 ? launch_tc_pair_t<256, EPI_SWIGLU>(p, grid, st)
                                          : launch_tc_pair_t<128, EPI_SWIGLU>(p, grid, st);
  if (epi == EPI_BF16) return bn == 256 ? launch_tc_pair_t<256, EPI_BF16>(p, grid, st)
                                        : launch_tc_pair_t<128, EPI_BF16>(p, grid, st);
  if (epi == EPI_F32) return bn == 256 ? launch_tc_pair_t<256, EPI_F32>(p, grid, st)
                                       : launch_tc_pair_t<128, EPI_F32>(p, grid, st);
  if (epi == EPI_SWIGLU_BWD) return bn == 256 ? launch_tc_pair_t<256, EPI_SWIGLU_BWD>(p, grid, st)
                                              : launch_tc_pair_t<128, EPI_SWIGLU_BWD>(p, grid, st);
  if (epi == EPI_DOWN3) return bn == 256 ? launch_tc_pair_t<256, EPI_DOWN3>(p, grid, st)
                                         : launch_tc_pair_t<128, EPI_DOWN3>(p, grid, st);
  return cudaErrorInvalidValue;
}

// Pair tile width for M rows and N columns: the widest of 256/128 dividing N whose 256-row tiles
// still give every pair of SMs one; 0 when N has no such width.
int pick_pair_bn(long long M, int N, int sms) {
  const long long mt = (M + 255) / 256;
  for (int bn = 256; bn >= 128; bn >>= 1)
    if (N % bn == 0 && mt * (N / bn) >= sms / 2) return bn;
  return N % 128 == 0 ? 128 : 0;
}

struct TopkArgs {
  const float* s;
  const float* b;
  int T, E, k;
  int *idx, *rank, *blkcnt, *counts32;
  float* gates;
  uint16_t* bins;
  int ld_bins;
  TopkRefine rf;
  uint32_t* status;
};

template <int NJ>
cudaError_t launch_topk_t(const TopkArgs& a, cudaStream_t st) {
  const int nblk = (a.T + kTokBlock - 1) / kTokBlock;
  const size_t smem = a.E * sizeof(uint32_t) + (a.bins ? (size_t)(a.E + 2) * kTokBlock * sizeof(uint16_t) : 0);
  if (smem > 48 * 1024) {
    static unsigned done = 0;
    cudaError_t e = ensure_smem_attr(topk_kernel<NJ>, 64 * 1024 + 4 * 1024 + 1024, done);
    if (e != cudaSuccess) return e;
  }
  return launch_k(topk_kernel<NJ>, dim3(nblk), dim3(32 * topk_warps(NJ)), smem, st, 1, a.s, a.b, a.T, a.E, a.k,
                  a.idx, a.gates,
                  a.rank, a.blkcnt, a.counts32, a.bins, a.ld_bins, a.rf, a.status);
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st) {
  const int nj = (a.E + 31) / 32;
  if (nj <= 1) return launch_topk_t<1>(a, st);
  if (nj <= 2) return launch_topk_t<2>(a, st);
  if (nj <= 4) return launch_topk_t<4>(a, st);
  if (nj <= 8) return launch_topk_t<8>(a, st);
  if (nj <= 16) return launch_topk_t<16>(a, st);
  return launch_topk_t<32>(a, st);
}

template <typename T>
cudaError_t launch_combine(const T* o, const float* gates, const int* prow, int T_, int k, int l, T* z,
                           cudaStream_t st) {
  const dim3 grid((T_ + 7) / 8), block(256);
  if (k <= 2) return launch_k(combine_kernel<T, 2>, grid, block, 0, st, 1, o, gates, prow, T_, k, l, z);
  if (k <= 4) return launch_k(combine_kernel<T, 4>, grid, block, 0, st, 1, o, gates, prow, T_, k, l, z);
  if (k <= 6) return launch_k(combine_kernel<T, 6>, grid, block, 0, st, 1, o, gates, prow, T_, k, l, z);
  return launch_k(combine_kernel<T, 8>, grid, block, 0, st, 1, o, gates, prow, T_, k, l, z);
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Stages timed by the optional per-stage profiler (lmoe_profile_enable).
enum Stage : int {
  ST_RMS = 0, ST_DOWN, ST_ROUTER, ST_K1, ST_TOPK, ST_PLAN, ST_GATHER, ST_HIST, ST_SHARED, ST_EXPERT1,
  ST_EXPERT2, ST_COMBINE, ST_UP, ST_QB_UPDATE, ST_COUNT
};
const char* const kStageNames[ST_COUNT] = {
    "rms", "down_proj", "router", "norm_down_router", "topk", "plan", "gather", "hist", "shared_swiglu",
    "expert_swiglu", "expert_down", "combine", "up_proj", "qb_update"};
constexpr int kProfRecords = 4096;

// One cached CUDA graph of a call with fixed arguments (see lmoe_forward).
struct GraphCache {
  cudaGraphExec_t exec = nullptr;
  const void* x = nullptr;
  void* y = nullptr;
  int T = -1;
  uint32_t flags = 0;
  float beta = 0.f;
  uint64_t state = 0;  // the statistics state the call started from (it decides the kernels)
  int seen = 0;
  long long kernels = 0;
  bool same(const void* x_, void* y_, int T_, uint32_t f_, float b_, uint64_t s_) const {
    return x == x_ && y == y_ && T == T_ && flags == f_ && beta == b_ && state == s_;
  }
  void reset(const void* x_, void* y_, int T_, uint32_t f_, float b_, uint64_t s_) {
    if (exec) cudaGraphExecDestroy(exec);
    exec = nullptr;
    x = x_;
    y = y_;
    T = T_;
    flags = f_;
    beta = b_;
    state = s_;
    seen = 0;
    kernels = 0;
  }
};

// Where the statistics of recorded forwards stand.  A recorded forward's score bins stay in one
// of two bin buffers, uncounted ("pending"), until the next lmoe_qb_update counts them into its
// histogram quantiles directly, or another recorded forward or lmoe_get_hist adds them to the
// accumulated histogram (hist_live: the accumulated rows may be non-zero).
struct StatsState {
  int pend_T = 0;      // tokens of the pending bins (0: none)
  int pend_buf = 0;    // bin buffer holding them
  bool hist_live = false;
  uint64_t key() const { return ((uint64_t)(uint32_t)pend_T << 2) | ((uint64_t)pend_buf << 1) | (hist_live ? 1u : 0u); }
};

struct ProfRecord {
  int first, n;                 // stages [first, first + n)
  cudaEvent_t ev[ST_COUNT + 1];  // ev[i] marks the start of stage first + i; ev[n] the end
};

}  // namespace

// ---------------------------------------------------------------------- handle
// Workspace of lmoe_forward_backward, allocated by its first call (sized for max_tokens).
struct BwdWork {
  void* mem = nullptr;
  bf16 *xh = nullptr, *ps = nullptr, *dps = nullptr, *dz = nullptr;  // token rows
  bf16 *pe = nullptr, *dpe = nullptr, *d_o = nullptr, *dhe = nullptr;  // padded expert rows
  bf16 *dlogit = nullptr, *dh = nullptr;
  float *dlp = nullptr, *dhr = nullptr, *dxh = nullptr, *gpart = nullptr;
  long long RP = 0;  // rows of the padded expert layout, a multiple of 128
  // maps of the padded expert-row buffers (fixed addresses)
  CUtensorMap pe_out, dpe_out, dpe_k, dpe_mn, do_k, do_mn, dhe_out, aperm_mn, act_mn;
  CUtensorMap ps_out;  // the shared expert's pre-activations [max_tokens, 2 hs]
};

struct lmoe_handle {
  lmoe_config cfg;
  int device = 0, sms = 148;
  size_t es = 2;  // bytes per activation element
  bool bf = true;
  bool unit_gain = true;
  int nblk_max = 0, max_mtiles = 0, ld_bins = 0;
  uint8_t* arena = nullptr;
  size_t arena_bytes = 0;
  // repacked weights; an fp32 layer keeps each as three bf16 parts along K ([.., 3K])
  void* w_down = nullptr;   // bf16 [l, d] or [l, 2d] (hi|lo); f32 [l, 3d]
  void* w_r = nullptr;      // [E_pad, 3l] (hi|mid|lo of the fp32 router)
  float* c = nullptr;       // [E]
  double* wc = nullptr;     // W_comb [E, d] fp64 (exact decision of ambiguous top-k)
  float tau = 0.f;          // near-tie width below which a token's top-k is decided in fp64
  void* ws13 = nullptr;     // [2hs, d] interleaved (f32: [2hs, 3d])
  void* w13 = nullptr;      // [E, 2h, l] interleaved (f32: [E, 2h, 3l])
  void* w2 = nullptr;       // [E, l, h] (f32: [E, l, 3h])
  void* wy = nullptr;       // [d, l + hs] (f32: [d, 3l + 3hs])
  // workspace
  float* r = nullptr;
  void* hx = nullptr;       // [Tm, 3l] (hi|mid|lo of h)
  float* s = nullptr;
  uint16_t* bins = nullptr;  // 2 x [E, ld_bins] histogram bin of every score, expert-major
  StatsState ss;
  int *idx = nullptr, *rank = nullptr, *blkcnt = nullptr, *blkbase = nullptr, *counts = nullptr;
  int* counts32 = nullptr;  // [32][E] partial counts of the top-k blocks
  bool counts32_dirty = true;
  int *offsets = nullptr, *num_mtiles = nullptr, *perm = nullptr, *inv = nullptr;
  int *pad_delta = nullptr, *prow = nullptr;  // padded expert layout of the grouped GEMMs
  long long rows_pad = 0;                     // rows of that layout (upper bound)
  float* gates = nullptr;
  int2* mtiles = nullptr;
  // MXFP8 routed experts: 8-bit elements and scale bytes of the weights, of h, of the gathered
  // rows and of the activations
  bool q8 = false;
  uint8_t *w13q = nullptr, *w13sf = nullptr, *w2q = nullptr, *w2sf = nullptr;
  uint8_t *hq = nullptr, *hsf = nullptr, *aq = nullptr, *aqsf = nullptr, *actq = nullptr, *actsf = nullptr;
  CUtensorMap tm_aq, tm_aq_part[3], tm_w13q, tm_actq, tm_actq_part[3], tm_w2q;
  void *a_perm = nullptr, *act = nullptr, *o = nullptr, *z = nullptr, *a_s = nullptr;
  void *x_stage = nullptr, *y_stage = nullptr;
  // lmoe_forward_host: two input staging buffers, so the next call's host-to-device copy (on its
  // own stream) overlaps this call's forward
  void* x_stage2 = nullptr;
  // fp32 layers: the three bf16 parts of x and of z for the split-precision products, and E
  // rounded up to 64 (the router's weight rows and column offsets are padded with zeros)
  void *x3 = nullptr, *z3 = nullptr;
  int E_pad = 0;
  CUtensorMap tm_x3, tm_z3;
  void* y_stage2 = nullptr;
  int host_slot = 0;
  cudaStream_t cp_in = nullptr;
  cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_fwd[2] = {nullptr, nullptr};
  bool fwd_recorded[2] = {false, false};
  // LMOE_ASYNC_OUTPUT: output copies on their own stream; out_pending[i] = an output copy from
  // staging slot i was enqueued there and no forward into that slot has waited for it yet
  cudaStream_t cp_out = nullptr;
  cudaEvent_t ev_out[2] = {nullptr, nullptr};
  bool out_pending[2] = {false, false};
  int last_out = -1;  // slot of the last output copy enqueued on cp_out
  // state
  float* bias = nullptr;
  uint32_t* hist = nullptr;
  long long* ntok = nullptr;
  long long* load = nullptr;  // [E] (token, slot) pairs routed to each expert since the last update
  uint32_t* status = nullptr;
  double* u = nullptr;
  unsigned int* qb_done = nullptr;  // block counter of the QB update kernel (zero between calls)
  int last_T = 0;
  // tensor maps (bf16)
  // weight maps of the non-grouped GEMMs exist for each tile width 64/128/256 that divides N
  CUtensorMap tm_hx, tm_aperm, tm_w13, tm_act, tm_w2, tm_z, tm_as, tm_o, tm_s;
  // A_perm, act and o with boxes of 32, 64 and 96 rows: the grouped GEMMs move only the valid
  // rows of an expert's last tile
  CUtensorMap tm_aperm_part[3], tm_act_part[3], tm_o_part[3];
  CUtensorMap tm_wr[3], tm_wdown[3], tm_ws13[3], tm_wy[3];
  bool fused_k1 = false;       // l <= 256 and E <= 256: RMSNorm + W_down + router in one kernel
  CUtensorMap tm_k1_wd, tm_k1_wr;        // boxes of the whole of l and E rows (one CTA per tile)
  CUtensorMap tm_k1_wd2, tm_k1_wr2;      // boxes of l/2 and E/2 rows (a cluster of two per tile)
  bool k1_split = false;                 // the two-CTA form exists (l % 128 == 0, E % 64 == 0)
  int bn_e1 = 256, bn_e2 = 256;
  // launch counter and optional per-stage profiler
  long long launches = 0;
  bool profiling = false;
  std::vector<ProfRecord> prof;
  int prof_used = 0;
  ProfRecord* cur = nullptr;
  // graph replay of repeated calls
  cudaStream_t cap = nullptr;
  GraphCache g_fwd[2], g_qb;  // two forward graphs (the host path alternates input buffers)
  // the backward of lmoe_forward_backward, and the buffers its graph was captured with besides x,
  // dy and the handle's own: the weights' and the gradients' pointers
  GraphCache g_bwd;
  const void* bwd_ptrs[23] = {};
  // LMOE_UPDATE_BIAS: the update's step and flags, and the branch it runs on
  bool upd_set = false;
  float upd_beta = 0.f;
  uint32_t upd_flags = 0;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  long long g_tick = 0;
  long long g_used[2] = {0, 0};
  BwdWork* bw = nullptr;
};

namespace {

struct Arena {
  size_t off = 0;
  std::vector<std::pair<void**, size_t>> items;
  void add(void** p, size_t bytes) {
    items.push_back({p, off});
    off += align_up(bytes ? bytes : 1, 1024);
  }
};

void plan_layout(lmoe_handle* h, Arena& a) {
  const lmoe_config& c = h->cfg;
  const size_t es = h->es;
  const size_t Tm = c.max_tokens, TK = (size_t)c.max_tokens * c.k;
  const size_t d = c.d, l = c.l, E = c.E, hh = c.h, hs = c.hs;
  // weights (an fp32 layer keeps every GEMM operand as three bf16 parts along K)
  const size_t Ep = (size_t)h->E_pad;
  a.add(&h->w_down, h->bf ? (h->unit_gain ? 1 : 2) * l * d * es : 3 * l * d * 2);
  a.add(&h->w_r, Ep * 3 * l * 2);
  a.add((void**)&h->c, Ep * 4);
  a.add((void**)&h->wc, E * d * 8);
  if (hs) a.add(&h->ws13, h->bf ? 2 * hs * d * es : 2 * hs * 3 * d * 2);
  if (h->q8) {
    a.add((void**)&h->w13q, 2 * E * hh * l);
    a.add((void**)&h->w13sf, 2 * E * hh * l / 32);
    a.add((void**)&h->w2q, E * l * hh);
    a.add((void**)&h->w2sf, E * l * hh / 32);
  } else {
    a.add(&h->w13, h->bf ? 2 * E * hh * l * es : 2 * E * hh * 3 * l * 2);
    a.add(&h->w2, h->bf ? E * l * hh * es : E * l * 3 * hh * 2);
  }
  a.add(&h->wy, h->bf ? d * (l + hs) * es : d * 3 * (l + hs) * 2);
  // workspace
  a.add((void**)&h->r, Tm * 4);
  a.add(&h->hx, Tm * 3 * l * 2);
  if (!h->bf) {
    a.add(&h->x3, Tm * 3 * d * 2);
    a.add(&h->z3, Tm * 3 * l * 2);
  }
  a.add((void**)&h->s, Tm * E * 4);
  a.add((void**)&h->bins, 2 * (size_t)h->ld_bins * E * 2);
  a.add((void**)&h->idx, TK * 4);
  a.add((void**)&h->gates, TK * 4);
  a.add((void**)&h->rank, TK * 4);
  a.add((void**)&h->blkcnt, (size_t)h->nblk_max * E * 4);
  a.add((void**)&h->blkbase, (size_t)h->nblk_max * E * 4);
  a.add((void**)&h->counts, E * 4);
  a.add((void**)&h->counts32, (size_t)kCountCopies * E * 4);
  a.add((void**)&h->offsets, (E + 1) * 4);
  a.add((void**)&h->num_mtiles, 4);
  a.add((void**)&h->mtiles, (size_t)h->max_mtiles * 8);
  a.add((void**)&h->perm, TK * 4);
  a.add((void**)&h->inv, TK * 4);
  a.add((void**)&h->prow, TK * 4);
  a.add((void**)&h->pad_delta, E * 4);
  const size_t RP = (size_t)h->rows_pad;
  if (h->q8) {
    a.add((void**)&h->hq, Tm * l);
    a.add((void**)&h->hsf, Tm * l / 32);
    a.add((void**)&h->aq, RP * l);
    const size_t RP128 = (RP + 127) / 128 * 128;  // scale atoms cover whole 128-row tiles
    a.add((void**)&h->aqsf, RP128 * l / 32);
    a.add((void**)&h->actq, RP * hh);
    a.add((void**)&h->actsf, RP128 * hh / 32);
  } else {
    a.add(&h->a_perm, h->bf ? RP * l * es : RP * 3 * l * 2);
    a.add(&h->act, h->bf ? RP * hh * es : RP * 3 * hh * 2);
  }
  a.add(&h->o, RP * l * es);
  a.add(&h->z, Tm * l * es);
  if (hs) a.add(&h->a_s, h->bf ? Tm * hs * es : Tm * 3 * hs * 2);
  a.add(&h->x_stage, Tm * d * es);
  a.add(&h->x_stage2, Tm * d * es);
  a.add(&h->y_stage, Tm * d * es);
  a.add(&h->y_stage2, Tm * d * es);
  // state
  a.add((void**)&h->bias, E * 4);
  a.add((void**)&h->hist, E * LMOE_NBINS * 4);
  a.add((void**)&h->ntok, 8);
  a.add((void**)&h->load, E * 8);
  a.add((void**)&h->status, 4);
  a.add((void**)&h->u, E * 8);
  a.add((void**)&h->qb_done, 4);
}

int validate(const lmoe_config* c) {
  if (!c) return LMOE_EINVAL;
  if (c->d <= 0 || c->l <= 0 || c->E <= 0 || c->k <= 0 || c->h <= 0 || c->hs < 0 || c->max_tokens <= 0)
    return LMOE_EINVAL;
  if (c->k > c->E || c->nbins != LMOE_NBINS || !(c->rms_eps >= 0.f)) return LMOE_EINVAL;
  if (c->dtype != LMOE_F32 && c->dtype != LMOE_BF16) return LMOE_EINVAL;
  if (c->d % 64 || c->l % 64 || c->h % 64 || c->hs % 64) return LMOE_EUNSUPPORTED;
  if (c->k > 32 || c->E > 1024) return LMOE_EUNSUPPORTED;
  if (c->dtype == LMOE_BF16 && c->E % 64) return LMOE_EUNSUPPORTED;
  if (c->dtype == LMOE_F32 && c->E % 32) return LMOE_EUNSUPPORTED;
  if ((long long)c->max_tokens * c->k > (1LL << 30)) return LMOE_EUNSUPPORTED;
  if (c->experts != LMOE_EXPERTS_BF16 && c->experts != LMOE_EXPERTS_MXFP8) return LMOE_EINVAL;
  if (c->experts == LMOE_EXPERTS_MXFP8 && (c->dtype != LMOE_BF16 || c->l % 128 || c->h % 128))
    return LMOE_EUNSUPPORTED;
  return LMOE_OK;
}

#define CK(x)                                 \
  do {                                        \
    if ((x) != cudaSuccess) return LMOE_ECUDA; \
  } while (0)

int grid_1d(long long n, int threads) {
  long long b = (n + threads - 1) / threads;
  return (int)(b > 65535 * 16 ? 65535 * 16 : (b < 1 ? 1 : b));
}

int bn_index(int bn) { return bn == 64 ? 0 : (bn == 128 ? 1 : 2); }

// Maps of one weight matrix [rows, cols] for every tile width that divides rows.
bool make_weight_maps(CUtensorMap (&m)[3], const void* base, long long rows, long long cols) {
  bool ok = true;
  for (int bn = 64; bn <= 256; bn <<= 1)
    if (rows % bn == 0) ok &= make_map(&m[bn_index(bn)], base, rows, cols, cols, bn);
  return ok;
}

int build_maps(lmoe_handle* h) {
  const lmoe_config& c = h->cfg;
  const long long Tm = c.max_tokens, TK = (long long)c.max_tokens * c.k;
  const long long d = c.d, l = c.l, E = c.E, hh = c.h, hs = c.hs;
  h->bn_e1 = (2 * c.h) % 256 == 0 ? 256 : 128;
  h->bn_e2 = pick_bn(c.l);
  bool ok = true;
  ok &= make_map(&h->tm_hx, h->hx, Tm, 3 * l, 3 * l, 128);
  ok &= make_weight_maps(h->tm_wr, h->w_r, E, 3 * l);
  ok &= make_weight_maps(h->tm_wdown, h->w_down, l, h->unit_gain ? d : 2 * d);
  if (hs) ok &= make_weight_maps(h->tm_ws13, h->ws13, 2 * hs, d);
  const long long RP = h->rows_pad;
  (void)TK;
  if (h->q8) {
    ok &= make_map_u8(&h->tm_aq, h->aq, RP, l, l, 128);
    ok &= make_map_u8(&h->tm_actq, h->actq, RP, hh, hh, 128);
    for (int i = 0; i < 3; ++i) {
      ok &= make_map_u8(&h->tm_aq_part[i], h->aq, RP, l, l, 32 * (i + 1));
      ok &= make_map_u8(&h->tm_actq_part[i], h->actq, RP, hh, hh, 32 * (i + 1));
    }
    ok &= make_map_u8(&h->tm_w13q, h->w13q, E * 2 * hh, l, l, 128);
    ok &= make_map_u8(&h->tm_w2q, h->w2q, E * l, hh, hh, 128);
  } else {
  ok &= make_map(&h->tm_aperm, h->a_perm, RP, l, l, 128);
  ok &= make_map(&h->tm_w13, h->w13, E * 2 * hh, l, l, h->bn_e1);
  ok &= make_map(&h->tm_act, h->act, RP, hh, hh, 128);
  ok &= make_map(&h->tm_o, h->o, RP, l, l, 128);
  for (int i = 0; i < 3; ++i) {
    ok &= make_map(&h->tm_aperm_part[i], h->a_perm, RP, l, l, 32 * (i + 1));
    ok &= make_map(&h->tm_act_part[i], h->act, RP, hh, hh, 32 * (i + 1));
    ok &= make_map(&h->tm_o_part[i], h->o, RP, l, l, 32 * (i + 1));
  }
  ok &= make_map(&h->tm_w2, h->w2, E * l, hh, hh, h->bn_e2);
  }
  ok &= make_map_f32(&h->tm_s, h->s, Tm, E, E, 128);
  ok &= make_map(&h->tm_z, h->z, Tm, l, l, 128);
  if (hs) ok &= make_map(&h->tm_as, h->a_s, Tm, hs, hs, 128);
  ok &= make_weight_maps(h->tm_wy, h->wy, d, l + hs);
  h->fused_k1 = c.l <= 256 && c.E <= 256;
  if (h->fused_k1) {
    ok &= make_map(&h->tm_k1_wd, h->w_down, l, h->unit_gain ? d : 2 * d, h->unit_gain ? d : 2 * d, (int)l);
    ok &= make_map(&h->tm_k1_wr, h->w_r, E, 3 * l, 3 * l, (int)E);
    h->k1_split = c.l % 128 == 0 && c.E % 64 == 0;
    if (h->k1_split) {
      ok &= make_map(&h->tm_k1_wd2, h->w_down, l, h->unit_gain ? d : 2 * d, h->unit_gain ? d : 2 * d, (int)l / 2);
      ok &= make_map(&h->tm_k1_wr2, h->w_r, E, 3 * l, 3 * l, (int)E / 2);
    }
  }
  return ok ? LMOE_OK : LMOE_ECUDA;
}

// Maps of an fp32 layer: every GEMM operand is three bf16 parts along K (weights split at create,
// x and z in each forward, h, a_s and act written that way by the epilogues); o and y are fp32.
int build_maps_f32(lmoe_handle* h) {
  const lmoe_config& c = h->cfg;
  const long long Tm = c.max_tokens, d = c.d, l = c.l, E = c.E, hh = c.h, hs = c.hs, Ep = h->E_pad;
  const long long RP = h->rows_pad;
  h->bn_e1 = (2 * c.h) % 256 == 0 ? 256 : 128;
  h->bn_e2 = pick_bn(c.l);
  bool ok = true;
  ok &= make_map(&h->tm_x3, h->x3, Tm, 3 * d, 3 * d, 128);
  ok &= make_weight_maps(h->tm_wdown, h->w_down, l, 3 * d);
  ok &= make_map(&h->tm_hx, h->hx, Tm, 3 * l, 3 * l, 128);
  ok &= make_weight_maps(h->tm_wr, h->w_r, Ep, 3 * l);
  ok &= make_map_f32(&h->tm_s, h->s, Tm, E, E, 128);
  if (hs) {
    ok &= make_weight_maps(h->tm_ws13, h->ws13, 2 * hs, 3 * d);
    ok &= make_map(&h->tm_as, h->a_s, Tm, 3 * hs, 3 * hs, 128);
  }
  ok &= make_map(&h->tm_aperm, h->a_perm, RP, 3 * l, 3 * l, 128);
  ok &= make_map(&h->tm_w13, h->w13, E * 2 * hh, 3 * l, 3 * l, h->bn_e1);
  ok &= make_map(&h->tm_act, h->act, RP, 3 * hh, 3 * hh, 128);
  ok &= make_map(&h->tm_w2, h->w2, E * l, 3 * hh, 3 * hh, h->bn_e2);
  ok &= make_map_f32(&h->tm_o, h->o, RP, l, l, 128);
  for (int i = 0; i < 3; ++i) {
    ok &= make_map(&h->tm_aperm_part[i], h->a_perm, RP, 3 * l, 3 * l, 32 * (i + 1));
    ok &= make_map(&h->tm_act_part[i], h->act, RP, 3 * hh, 3 * hh, 32 * (i + 1));
    ok &= make_map_f32(&h->tm_o_part[i], h->o, RP, l, l, 32 * (i + 1));
  }
  ok &= make_map(&h->tm_z3, h->z3, Tm, 3 * l, 3 * l, 128);
  ok &= make_weight_maps(h->tm_wy, h->wy, d, 3 * (l + hs));
  return ok ? LMOE_OK : LMOE_ECUDA;
}

// Profiler: opens a record for stages [first, first + n) of one call, marks stage starts, closes.
void prof_open(lmoe_handle* h, int first, int n) {
  h->cur = nullptr;
  if (!h->profiling || h->prof_used >= kProfRecords) return;
  if ((int)h->prof.size() <= h->prof_used) {
    ProfRecord r;
    r.first = r.n = 0;
    for (auto& e : r.ev) cudaEventCreate(&e);
    h->prof.push_back(r);
  }
  h->cur = &h->prof[h->prof_used++];
  h->cur->first = first;
  h->cur->n = n;
}
void mark(lmoe_handle* h, int stage, cudaStream_t st) {
  if (h->cur) cudaEventRecord(h->cur->ev[stage - h->cur->first], st);
}
void prof_close(lmoe_handle* h, cudaStream_t st) {
  if (h->cur) cudaEventRecord(h->cur->ev[h->cur->n], st);
  h->cur = nullptr;
}

TcParams tc_base(lmoe_handle* h) {
  TcParams p;
  memset(&p, 0, sizeof(p));
  p.status = h->status;
  return p;
}

// ---- stages shared by lmoe_forward and lmoe_route_scores
uint16_t* bin_buffer(lmoe_handle* h, int i) { return h->bins + (size_t)i * h->ld_bins * h->cfg.E; }

// State after a routing of T tokens with `flags` that started from `pre`.
StatsState after_routing(const StatsState& pre, int T, uint32_t flags) {
  StatsState post = pre;
  if (flags & LMOE_RECORD_STATS) {
    if (pre.pend_T) post.hist_live = true;
    post.pend_buf = pre.pend_T ? pre.pend_buf ^ 1 : pre.pend_buf;
    post.pend_T = T;
  }
  return post;
}

// Adds pending bins (pend_T tokens, buffer buf) to the accumulated histogram and N.
int flush_bins(lmoe_handle* h, int pend_T, int buf, cudaStream_t st) {
  CK(launch_k(hist_kernel, dim3(h->cfg.E), dim3(kHistThreads), 0, st, 1, (const uint16_t*)bin_buffer(h, buf),
              h->ld_bins, pend_T, h->hist, h->ntok));
  h->launches += 1;
  return LMOE_OK;
}

// The bias update (QB, or the sign rule) from the statistics state `at`.  `pdl` = false launches
// it without programmatic serialisation: on a side branch its blocks would otherwise become
// resident as soon as the kernel before the fork allowed dependents, and sit in their wait
// holding SM slots that the persistent GEMMs of the main branch need.
int launch_qb(lmoe_handle* h, float beta, uint32_t flags, const StatsState& at, cudaStream_t s, bool pdl = true) {
  const int literal = (flags & LMOE_QB_LITERAL) ? 1 : 0, sign = (flags & LMOE_BIAS_SIGN) ? 1 : 0;
  const uint16_t* bins = (const uint16_t*)bin_buffer(h, at.pend_buf);
  if (pdl) {
    CK(launch_k(qb_update_kernel, dim3(h->cfg.E), dim3(kQbThreads), 0, s, 1, h->hist, h->ntok, h->load, h->bias,
                h->cfg.E, h->cfg.k, literal, sign, beta, h->u, h->qb_done, bins, h->ld_bins, at.pend_T,
                at.hist_live ? 1 : 0, h->status));
  } else {
    qb_update_kernel<<<h->cfg.E, kQbThreads, 0, s>>>(h->hist, h->ntok, h->load, h->bias, h->cfg.E, h->cfg.k,
                                                     literal, sign, beta, h->u, h->qb_done, bins, h->ld_bins,
                                                     at.pend_T, at.hist_live ? 1 : 0, h->status);
    CK(cudaGetLastError());
  }
  h->launches += 1;
  return LMOE_OK;
}

// LMOE_UPDATE_BIAS without profiling: the update is a branch that forks off `st` once every
// statistic it reads is final and joins `st` at the end of the forward (no later kernel of the
// forward reads or writes the bias or the statistics).  QB reads the histogram, N and the bins
// that top-k writes, so it forks right after top-k, beside the latency-bound plan kernel, unless
// bins of an earlier forward still have to be flushed into the histogram; the plan kernel then
// leaves the loads alone (the update zeroes them, as it would after adding them).  The sign rule
// reads the loads that the plan kernel adds, so it forks after routing.
bool fork_after_topk(lmoe_handle* h, uint32_t flags, const StatsState& pre) {
  return !(h->upd_flags & LMOE_BIAS_SIGN) && !pre.pend_T && (flags & LMOE_UPDATE_BIAS) && !h->profiling;
}
int fork_update(lmoe_handle* h, int T, uint32_t flags, const StatsState& pre, cudaStream_t st) {
  if (!(flags & LMOE_UPDATE_BIAS) || h->profiling) return LMOE_OK;
  CK(cudaEventRecord(h->ev_fork, st));
  CK(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
  int rc = launch_qb(h, h->upd_beta, h->upd_flags, after_routing(pre, T, flags), h->side, false);
  if (rc) return rc;
  CK(cudaEventRecord(h->ev_join, h->side));
  return LMOE_OK;
}
int join_update(lmoe_handle* h, uint32_t flags, cudaStream_t st) {
  if (!(flags & LMOE_UPDATE_BIAS) || h->profiling) return LMOE_OK;
  CK(cudaStreamWaitEvent(st, h->ev_join, 0));
  return LMOE_OK;
}

int route_from_scores(lmoe_handle* h, int T, uint32_t flags, const StatsState& pre, const void* x,
                      cudaStream_t st) {
  const StatsState post = after_routing(pre, T, flags);
  const lmoe_config& c = h->cfg;
  const int nblk = (T + kTokBlock - 1) / kTokBlock;
  mark(h, ST_TOPK, st);
  // the count copies are zero between routings (the gather kernel clears them after the plan
  // kernel has read them) unless an earlier routing stopped half-way
  if (h->counts32_dirty) CK(cudaMemsetAsync(h->counts32, 0, (size_t)kCountCopies * c.E * sizeof(int), st));
  h->counts32_dirty = true;
  TopkArgs ta{h->s, h->bias, T, c.E, c.k, h->idx, h->rank, h->blkcnt, h->counts32, h->gates,
              (flags & LMOE_RECORD_STATS) ? bin_buffer(h, post.pend_buf) : nullptr, h->ld_bins,
              TopkRefine{x, h->bf ? 1 : 0, c.d, h->wc, h->c, c.rms_eps, h->tau}, h->status};
  CK(launch_topk(ta, st));
  const bool early = fork_after_topk(h, flags, pre);
  if (early) {
    int rc = fork_update(h, T, flags, pre, st);
    if (rc) return rc;
  }
  mark(h, ST_PLAN, st);
  CK(launch_k(plan_kernel, dim3((c.E + kPlanExperts - 1) / kPlanExperts), dim3(1024), 0, st, 1, (const int*)h->counts32, h->counts,
              (const int*)h->blkcnt, nblk, c.E, h->offsets, h->pad_delta, h->blkbase, h->mtiles, h->num_mtiles,
              // an update already forked clears the loads itself, which equals adding them first
              ((flags & LMOE_RECORD_STATS) && !early) ? h->load : (long long*)nullptr));
  const int pairs = T * c.k;
  const dim3 ggrid((pairs + 8 * kGatherPairs - 1) / (8 * kGatherPairs));
  int4* clear = reinterpret_cast<int4*>(h->counts32);
  const int nclear = kCountCopies * c.E / 4;
  mark(h, ST_GATHER, st);
  if (h->bf) {
    CK(launch_k(gather_kernel<bf16>, ggrid, dim3(256), 0, st, 1, (const bf16*)h->hx, 3 * c.l, c.l,
                (const int*)h->idx, (const int*)h->rank, (const int*)h->blkbase, (const int*)h->pad_delta, T, c.E,
                c.k, h->perm, h->inv, h->prow, (bf16*)h->a_perm, clear, nclear, h->status));
    if (h->q8 && x) {
      // MXFP8 experts: h (fp32, from its hi | mid | lo parts) quantised once per token, then each
      // pair's 8-bit row and scale bytes copied into the padded expert layout
      CK(launch_k(mx_quant_rows_kernel, dim3(grid_1d((long long)T * c.l / 32, 256)), dim3(256), 0, st, 1,
                  (const bf16*)h->hx, 3, (long long)T, c.l, h->hq, h->hsf, 0));
      CK(launch_k(gather_q8_kernel, dim3((pairs + 7) / 8), dim3(256), 0, st, 1, (const uint8_t*)h->hq,
                  (const uint8_t*)h->hsf, c.l, (const int*)h->prow, pairs, c.k, h->aq, h->aqsf));
      h->launches += 2;
    }
  } else {
    // fp32 layer: all three parts of h travel with each row (the experts' split-precision products)
    CK(launch_k(gather_kernel<bf16>, ggrid, dim3(256), 0, st, 1, (const bf16*)h->hx, 3 * c.l, 3 * c.l,
                (const int*)h->idx, (const int*)h->rank, (const int*)h->blkbase, (const int*)h->pad_delta, T, c.E,
                c.k, h->perm, h->inv, h->prow, (bf16*)h->a_perm, clear, nclear, h->status));
  }
  h->counts32_dirty = false;
  mark(h, ST_HIST, st);
  h->launches += 3;
  // the bins of an earlier recorded forward that no update has counted yet join the histogram
  // before their buffer is reused (this forward's own bins stay pending for lmoe_qb_update)
  if ((flags & LMOE_RECORD_STATS) && pre.pend_T) {
    int rc = flush_bins(h, pre.pend_T, pre.pend_buf, st);
    if (rc) return rc;
  }
  h->last_T = T;
  return early ? LMOE_OK : fork_update(h, T, flags, pre, st);
}

int forward_bf16(lmoe_handle* h, const void* x, void* y, int T, uint32_t flags, const StatsState& pre,
                 cudaStream_t st, bool save_pre = false) {
  const lmoe_config& c = h->cfg;
  const int mt = (T + 127) / 128;
  CUtensorMap tm_x;
  if (!make_map(&tm_x, x, T, c.d, c.d, 128)) return LMOE_EINVAL;
  mark(h, ST_RMS, st);
  if (h->fused_k1) {
    mark(h, ST_DOWN, st);
    mark(h, ST_ROUTER, st);
    mark(h, ST_K1, st);
    // a cluster of two CTAs per tile while the tiles fill at most half of the SMs
    const int ns = (h->k1_split && 2 * mt <= h->sms) ? 2 : 1;
    K1Params kp;
    memset(&kp, 0, sizeof(kp));
    kp.tm_s = h->tm_s;
    kp.tm_x = tm_x;
    kp.tm_wd = ns == 2 ? h->tm_k1_wd2 : h->tm_k1_wd;
    kp.tm_hx = h->tm_hx;
    kp.tm_wr = ns == 2 ? h->tm_k1_wr2 : h->tm_k1_wr;
    kp.ns = ns;
    kp.T = T;
    kp.d = c.d;
    kp.l = c.l;
    kp.E = c.E;
    kp.wd_segments = h->unit_gain ? 1 : 2;
    kp.eps = c.rms_eps;
    kp.r = h->r;
    kp.c = h->c;
    kp.status = h->status;
    static unsigned done = 0;
    CK(ensure_smem_attr(k1_kernel, kK1SmemBytes, done));
    CK(launch_k(k1_kernel, dim3(ns * std::min(mt, h->sms / ns)), dim3(kTcThreads), kK1SmemBytes, st, ns, kp));
    h->launches += 1;
  } else {
    CK(launch_k(rms_kernel<bf16>, dim3((T + 7) / 8), dim3(256), 0, st, 1, (const bf16*)x, T, c.d, c.rms_eps, h->r));
    // h = r * (x Wdown^T), stored as hi | mid | lo bf16 parts
    mark(h, ST_DOWN, st);
    {
      TcParams p = tc_base(h);
      p.tmA[0] = tm_x;
      p.tmA[1] = tm_x;
      p.nseg = h->unit_gain ? 1 : 2;
      p.seg[0] = {0, 0, 0, c.d / 64};
      p.seg[1] = {0, 0, c.d, c.d / 64};
      p.M = T;
      p.M_rows = T;
      p.tmOut = h->tm_hx;
      p.split = c.l;
      p.row_scale = h->r;
      // two-CTA tiles for long token batches: at the wide layer (K = d = 7168) 0.37-0.40 ms against
      // 0.42-0.45 ms on single-CTA tiles
      const int pbn = T >= 256 * 8 ? pick_pair_bn(T, c.l, h->sms) : 0;
      if (pbn) {  // each CTA loads BN/2 rows of W_down
        p.tmB = h->tm_wdown[bn_index(pbn / 2)];
        p.n_tiles = c.l / pbn;
        p.band_n = pick_band(p.n_tiles, pbn, (h->unit_gain ? 1 : 2) * (long long)c.d);
        const int tiles = (T + 255) / 256 * p.n_tiles;
        CK(launch_tc_pair(p, EPI_DOWN3, pbn, 2 * std::min(tiles, h->sms / 2), st));
      } else {
        const int bn = pick_bn_for(T, c.l, h->sms, 64);
        p.tmB = h->tm_wdown[bn_index(bn)];
        p.n_tiles = c.l / bn;
        p.band_n = pick_band(p.n_tiles, bn, (h->unit_gain ? 1 : 2) * (long long)c.d);
        CK(launch_tc(p, EPI_DOWN3, bn, std::min(mt * p.n_tiles, h->sms), st));
      }
    }
    // s = sigmoid(h Wr^T + c) from six bf16 x bf16 products of the hi/mid/lo parts, walked chunk
    // by chunk over the three parts (the engine's split-router mode; tiles at most 128 wide)
    mark(h, ST_ROUTER, st);
    {
      TcParams p = tc_base(h);
      p.tmA[0] = h->tm_hx;
      p.tmA[1] = h->tm_hx;
      const int bn = std::min(pick_bn_for(T, c.E, h->sms, 64), 128);
      p.tmB = h->tm_wr[bn_index(bn)];
      const int L = c.l, nk = c.l / 64;
      p.nseg = 3;
      p.seg[0] = {0, 0, 0, nk};          // hi parts
      p.seg[1] = {0, L, L, nk};          // mid parts
      p.seg[2] = {0, 2 * L, 2 * L, nk};  // lo parts
      p.M = T;
      p.M_rows = T;
      p.n_tiles = c.E / bn;
      p.tmOut = h->tm_s;
      p.col_bias = h->c;
      CK(launch_tc(p, EPI_ROUTER, bn, std::min(mt * p.n_tiles, h->sms), st));
    }
    mark(h, ST_K1, st);
    h->launches += 3;
  }
  int rc = route_from_scores(h, T, flags, pre, x, st);
  if (rc) return rc;
  // shared expert, first half: a_s = silu(r x Ws1^T) * (r x Ws3^T)
  mark(h, ST_SHARED, st);
  if (c.hs) {
    TcParams p = tc_base(h);
    p.tmA[0] = tm_x;
    p.tmA[1] = tm_x;
    p.nseg = 1;
    p.seg[0] = {0, 0, 0, c.d / 64};
    p.M = T;
    p.M_rows = T;
    p.tmOut = h->tm_as;
    p.row_scale = h->r;
    if (save_pre) {  // a training step: the backward reads the pre-activations
      p.out_pre = 1;
      p.tmOut2 = h->bw->ps_out;
    }
    const int pbn = T >= 256 * 8 ? pick_pair_bn(T, 2 * c.hs, h->sms) : 0;
    if (pbn) {  // two-CTA tiles: each CTA loads BN/2 rows of the weights
      p.tmB = h->tm_ws13[bn_index(pbn / 2)];
      p.n_tiles = 2 * c.hs / pbn;
      p.band_n = pick_band(p.n_tiles, pbn, c.d);
      const int tiles = (T + 255) / 256 * p.n_tiles;
      CK(launch_tc_pair(p, EPI_SWIGLU, pbn, 2 * std::min(tiles, h->sms / 2), st));
    } else {
      const int bn = pick_bn_for(T, 2 * c.hs, h->sms, 128);
      p.tmB = h->tm_ws13[bn_index(bn)];
      p.n_tiles = 2 * c.hs / bn;
      p.band_n = pick_band(p.n_tiles, bn, c.d);
      CK(launch_tc(p, EPI_SWIGLU, bn, std::min(mt * p.n_tiles, h->sms), st));
    }
  }
  // routed experts, grouped over the permuted rows
  mark(h, ST_EXPERT1, st);
  if (h->q8) {
    static unsigned done1 = 0, done2 = 0;
    CK(ensure_smem_attr(q8_gemm_kernel<Q8_SWIGLU>, kQ8SmemBytes, done1));
    CK(ensure_smem_attr(q8_gemm_kernel<Q8_BF16>, kQ8SmemBytes, done2));
    Q8Params p;
    memset(&p, 0, sizeof(p));
    p.status = h->status;
    p.mtile_table = h->mtiles;
    p.num_mtiles = h->num_mtiles;
    // act (MXFP8) = silu(A W1_e^T) * (A W3_e^T)
    p.tmA = h->tm_aq;
    for (int i = 0; i < 3; ++i) p.tmA_part[i] = h->tm_aq_part[i];
    p.tmB = h->tm_w13q;
    p.a_sf = h->aqsf;
    p.b_sf = h->w13sf;
    p.n_tiles = 2 * c.h / 128;
    p.b_rows = 2 * c.h;
    p.nkb = c.l / 128;
    p.out_q = h->actq;
    p.out_sf = h->actsf;
    p.n_out = c.h;
    CK(launch_k(q8_gemm_kernel<Q8_SWIGLU>, dim3(h->sms), dim3(kQ8Threads), kQ8SmemBytes, st, 1, p));
    mark(h, ST_EXPERT2, st);
    // o (bf16) = act W2_e^T
    p.tmA = h->tm_actq;
    for (int i = 0; i < 3; ++i) p.tmA_part[i] = h->tm_actq_part[i];
    p.tmB = h->tm_w2q;
    p.a_sf = h->actsf;
    p.b_sf = h->w2sf;
    p.n_tiles = c.l / 128;
    p.b_rows = c.l;
    p.nkb = c.h / 128;
    p.out_q = nullptr;
    p.out_sf = nullptr;
    p.out_bf = (bf16*)h->o;
    p.n_out = c.l;
    CK(launch_k(q8_gemm_kernel<Q8_BF16>, dim3(h->sms), dim3(kQ8Threads), kQ8SmemBytes, st, 1, p));
  } else {
    {
    TcParams p = tc_base(h);
    p.tmA[0] = h->tm_aperm;
    p.tmA[1] = h->tm_aperm;
    p.tmB = h->tm_w13;
    p.nseg = 1;
    p.seg[0] = {0, 0, 0, c.l / 64};
    p.grouped = 1;
    p.n_tiles = 2 * c.h / h->bn_e1;
    p.mtile_table = h->mtiles;
    p.num_mtiles = h->num_mtiles;
    p.b_rows_per_group = 2 * c.h;
    p.tmOut = h->tm_act;
    p.trim = 1;
    for (int i = 0; i < 3; ++i) {
      p.tmA_part[i] = h->tm_aperm_part[i];
      p.tmOut_part[i] = h->tm_act_part[i];
    }
    // no evict-first hint on the weights: each expert's slice serves its few row tiles, which run
    // at about the same time, and the hint lost it from L2 before the last of them (measured:
    // the wide layer's step 6.3 -> 5.8 ms without the hints on both expert products)
    p.hint_out = 1;  // act is read by the next GEMM
    if (save_pre) {
      p.out_pre = 1;
      p.tmOut2 = h->bw->pe_out;
      p.trim = 0;
    }
    CK(launch_tc(p, EPI_SWIGLU, h->bn_e1, h->sms, st));
    }
    mark(h, ST_EXPERT2, st);
    TcParams p = tc_base(h);
    p.tmA[0] = h->tm_act;
    p.tmA[1] = h->tm_act;
    p.tmB = h->tm_w2;
    p.nseg = 1;
    p.seg[0] = {0, 0, 0, c.h / 64};
    p.grouped = 1;
    p.n_tiles = c.l / h->bn_e2;
    p.mtile_table = h->mtiles;
    p.num_mtiles = h->num_mtiles;
    p.b_rows_per_group = c.l;
    p.tmOut = h->tm_o;
    p.trim = 1;
    for (int i = 0; i < 3; ++i) {
      p.tmA_part[i] = h->tm_act_part[i];
      p.tmOut_part[i] = h->tm_o_part[i];
    }
    p.hint_out = 1;  // o is read by the combine kernel
    CK(launch_tc(p, EPI_BF16, h->bn_e2, h->sms, st));
  }
  mark(h, ST_COMBINE, st);
  CK(launch_combine((const bf16*)h->o, h->gates, h->prow, T, c.k, c.l, (bf16*)h->z, st));
  // y = [z | a_s] [W_up | Ws2]^T
  mark(h, ST_UP, st);
  {
    TcParams p = tc_base(h);
    p.tmA[0] = h->tm_z;
    p.tmA[1] = c.hs ? h->tm_as : h->tm_z;
    p.nseg = c.hs ? 2 : 1;
    p.seg[0] = {0, 0, 0, c.l / 64};
    p.seg[1] = {1, 0, c.l, c.hs / 64};
    p.M = T;
    p.M_rows = T;
    if (!make_map(&p.tmOut, y, T, c.d, c.d, 128)) return LMOE_EINVAL;
    const int pbn = T >= 256 * 8 ? pick_pair_bn(T, c.d, h->sms) : 0;
    if (pbn) {
      p.tmB = h->tm_wy[bn_index(pbn / 2)];
      p.n_tiles = c.d / pbn;
      p.band_n = pick_band(p.n_tiles, pbn, c.l + c.hs);
      const int tiles = (T + 255) / 256 * p.n_tiles;
      CK(launch_tc_pair(p, EPI_BF16, pbn, 2 * std::min(tiles, h->sms / 2), st));
    } else {
      const int bn = pick_bn_for(T, c.d, h->sms, 64);
      p.tmB = h->tm_wy[bn_index(bn)];
      p.n_tiles = c.d / bn;
      p.band_n = pick_band(p.n_tiles, bn, c.l + c.hs);
      CK(launch_tc(p, EPI_BF16, bn, std::min(mt * p.n_tiles, h->sms), st));
    }
  }
  h->launches += (c.hs ? 1 : 0) + 4;
  return join_update(h, flags, st);
}

// The six significant products of A = [hi | mid | lo] and B = [hi | mid | lo] (three bf16 parts of
// fp32 values along K each): part pairs (a, b), smallest first, as K segments of the engine.
constexpr int kSplitA[6] = {1, 2, 0, 1, 0, 0}, kSplitB[6] = {1, 0, 2, 0, 1, 0};
void split_segments(TcParams& p, int first, int a_map, int b_off, int K) {
  for (int i = 0; i < 6; ++i) p.seg[first + i] = KSeg{a_map, kSplitA[i] * K, b_off + kSplitB[i] * K, K / 64};
}

// fp32 layer: the same stages as forward_bf16, every product split-precision on the tensor cores.
int forward_f32(lmoe_handle* h, const void* xv, void* yv, int T, uint32_t flags, const StatsState& pre,
                cudaStream_t st) {
  const lmoe_config& c = h->cfg;
  const float* x = (const float*)xv;
  const int mt = (T + 127) / 128;
  const int d = c.d, l = c.l, hh = c.h, hs = c.hs;
  mark(h, ST_RMS, st);
  CK(launch_k(rms_kernel<float>, dim3((T + 7) / 8), dim3(256), 0, st, 1, x, T, d, c.rms_eps, h->r));
  CK(launch_k(split3_kernel, dim3(grid_1d((long long)T * d, 256)), dim3(256), 0, st, 1, x, (const float*)nullptr, T, d,
              (bf16*)h->x3, 3 * d, 0));
  mark(h, ST_DOWN, st);
  {  // h = r * (x W_down'^T), stored as hi | mid | lo parts
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = h->tm_x3;
    const int bn = pick_bn_for(T, l, h->sms, 64);
    p.tmB = h->tm_wdown[bn_index(bn)];
    p.nseg = 6;
    split_segments(p, 0, 0, 0, d);
    p.M = T;
    p.M_rows = T;
    p.n_tiles = l / bn;
    p.tmOut = h->tm_hx;
    p.split = l;
    p.row_scale = h->r;
    CK(launch_tc(p, EPI_DOWN3, bn, std::min(mt * p.n_tiles, h->sms), st));
  }
  mark(h, ST_ROUTER, st);
  {  // s = sigmoid(h W_r^T + c), chunk by chunk over the three parts (the engine's split-router mode)
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = h->tm_hx;
    const int bn = std::min(pick_bn_for(T, h->E_pad, h->sms, 64), 128);
    p.tmB = h->tm_wr[bn_index(bn)];
    const int nk = l / 64;
    p.nseg = 3;
    p.seg[0] = {0, 0, 0, nk};
    p.seg[1] = {0, l, l, nk};
    p.seg[2] = {0, 2 * l, 2 * l, nk};
    p.M = T;
    p.M_rows = T;
    p.n_tiles = h->E_pad / bn;
    p.tmOut = h->tm_s;
    p.col_bias = h->c;
    CK(launch_tc(p, EPI_ROUTER, bn, std::min(mt * p.n_tiles, h->sms), st));
  }
  mark(h, ST_K1, st);
  h->launches += 4;
  int rc = route_from_scores(h, T, flags, pre, xv, st);
  if (rc) return rc;
  mark(h, ST_SHARED, st);
  if (hs) {  // a_s = silu(r x Ws1'^T) * (r x Ws3'^T), stored as three parts
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = h->tm_x3;
    const int bn = pick_bn_for(T, 2 * hs, h->sms, 128);
    p.tmB = h->tm_ws13[bn_index(bn)];
    p.nseg = 6;
    split_segments(p, 0, 0, 0, d);
    p.M = T;
    p.M_rows = T;
    p.n_tiles = 2 * hs / bn;
    p.tmOut = h->tm_as;
    p.split = hs;
    p.row_scale = h->r;
    CK(launch_tc(p, EPI_SWIGLU3, bn, std::min(mt * p.n_tiles, h->sms), st));
  }
  mark(h, ST_EXPERT1, st);
  {  // act = silu(A W1_e^T) * (A W3_e^T) over each expert's rows, stored as three parts
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = h->tm_aperm;
    p.tmB = h->tm_w13;
    p.nseg = 6;
    split_segments(p, 0, 0, 0, l);
    p.grouped = 1;
    p.n_tiles = 2 * hh / h->bn_e1;
    p.mtile_table = h->mtiles;
    p.num_mtiles = h->num_mtiles;
    p.b_rows_per_group = 2 * hh;
    p.tmOut = h->tm_act;
    p.split = hh;
    p.trim = 1;
    for (int i = 0; i < 3; ++i) {
      p.tmA_part[i] = h->tm_aperm_part[i];
      p.tmOut_part[i] = h->tm_act_part[i];
    }
    CK(launch_tc(p, EPI_SWIGLU3, h->bn_e1, h->sms, st));
  }
  mark(h, ST_EXPERT2, st);
  {  // o = act W2_e^T, fp32
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = h->tm_act;
    p.tmB = h->tm_w2;
    p.nseg = 6;
    split_segments(p, 0, 0, 0, hh);
    p.grouped = 1;
    p.n_tiles = l / h->bn_e2;
    p.mtile_table = h->mtiles;
    p.num_mtiles = h->num_mtiles;
    p.b_rows_per_group = l;
    p.tmOut = h->tm_o;
    p.trim = 1;
    for (int i = 0; i < 3; ++i) {
      p.tmA_part[i] = h->tm_act_part[i];
      p.tmOut_part[i] = h->tm_o_part[i];
    }
    CK(launch_tc(p, EPI_F32, h->bn_e2, h->sms, st));
  }
  mark(h, ST_COMBINE, st);
  CK(launch_combine((const float*)h->o, h->gates, h->prow, T, c.k, l, (float*)h->z, st));
  CK(launch_k(split3_kernel, dim3(grid_1d((long long)T * l, 256)), dim3(256), 0, st, 1, (const float*)h->z,
              (const float*)nullptr, T, l, (bf16*)h->z3, 3 * l, 0));
  mark(h, ST_UP, st);
  {  // y = [z | a_s] [W_up | Ws2]^T: six part products of z, then six of a_s
    TcParams p = tc_base(h);
    p.tmA[0] = h->tm_z3;
    p.tmA[1] = hs ? h->tm_as : h->tm_z3;
    p.nseg = hs ? 12 : 6;
    split_segments(p, 0, 0, 0, l);
    if (hs) split_segments(p, 6, 1, 3 * l, hs);
    p.M = T;
    p.M_rows = T;
    if (!make_map_f32(&p.tmOut, yv, T, d, d, 128)) return LMOE_EINVAL;
    const int bn = pick_bn_for(T, d, h->sms, 64);
    p.tmB = h->tm_wy[bn_index(bn)];
    p.n_tiles = d / bn;
    CK(launch_tc(p, EPI_F32, bn, std::min(mt * p.n_tiles, h->sms), st));
  }
  h->launches += (hs ? 1 : 0) + 5;
  return join_update(h, flags, st);
}

int repack(lmoe_handle* h, const lmoe_weights* w, cudaStream_t st) {
  const lmoe_config& c = h->cfg;
  const long long d = c.d, l = c.l, E = c.E, hh = c.h, hs = c.hs;
  const int TPB = 256;
  if (h->bf) {
    const bf16* g = h->unit_gain ? nullptr : (const bf16*)w->rms_gain;
    if (h->unit_gain)
      fold_gain_kernel<bf16><<<grid_1d(l * d, TPB), TPB, 0, st>>>((const bf16*)w->w_down, nullptr, l, d,
                                                                  (bf16*)h->w_down, d, 0);
    else
      fold_gain_split_kernel<<<grid_1d(l * d, TPB), TPB, 0, st>>>((const bf16*)w->w_down, g, l, d,
                                                                  (bf16*)h->w_down);
    split3_kernel<<<grid_1d(E * l, TPB), TPB, 0, st>>>(w->w_router, nullptr, (int)E, (int)l, (bf16*)h->w_r,
                                                       (int)(3 * l), 0);
    if (hs)
      interleave_kernel<bf16><<<grid_1d(hs * d, TPB), TPB, 0, st>>>((const bf16*)w->ws1, (const bf16*)w->ws3, g, 1,
                                                                    hs, d, (bf16*)h->ws13);
    if (h->q8) {
      mx_quant_w13_kernel<<<grid_1d(2 * E * hh * l / 32, TPB), TPB, 0, st>>>(
          (const bf16*)w->w1, (const bf16*)w->w3, (int)E, (int)hh, (int)l, h->w13q, h->w13sf);
      mx_quant_rows_kernel<<<grid_1d(E * l * hh / 32, TPB), TPB, 0, st>>>((const bf16*)w->w2, 1, E * l, (int)hh,
                                                                         h->w2q, h->w2sf, 1);
    } else
      interleave_kernel<bf16><<<grid_1d(E * hh * l, TPB), TPB, 0, st>>>((const bf16*)w->w1, (const bf16*)w->w3,
                                                                        nullptr, E, hh, l, (bf16*)h->w13);
    if (!h->q8) CK(cudaMemcpyAsync(h->w2, w->w2, E * l * hh * 2, cudaMemcpyDeviceToDevice, st));
    fold_gain_kernel<bf16><<<grid_1d(d * l, TPB), TPB, 0, st>>>((const bf16*)w->w_up, nullptr, d, l,
                                                                (bf16*)h->wy, l + hs, 0);
    if (hs)
      fold_gain_kernel<bf16><<<grid_1d(d * hs, TPB), TPB, 0, st>>>((const bf16*)w->ws2, nullptr, d, hs,
                                                                   (bf16*)h->wy, l + hs, l);
  } else {
    // every GEMM operand as three bf16 parts along K (the gain folded into W_down and Ws1/Ws3 in
    // fp32 first); the router weights padded to E_pad rows of zeros
    const float* g = (const float*)w->rms_gain;
    split3_kernel<<<grid_1d(l * d, TPB), TPB, 0, st>>>((const float*)w->w_down, g, (int)l, (int)d, (bf16*)h->w_down,
                                                       (int)(3 * d), 0);
    CK(cudaMemsetAsync(h->w_r, 0, (size_t)h->E_pad * 3 * l * 2, st));
    split3_kernel<<<grid_1d(E * l, TPB), TPB, 0, st>>>(w->w_router, nullptr, (int)E, (int)l, (bf16*)h->w_r,
                                                       (int)(3 * l), 0);
    if (hs)
      interleave_split3_kernel<<<grid_1d(hs * d, TPB), TPB, 0, st>>>((const float*)w->ws1, (const float*)w->ws3, g, 1,
                                                                     (int)hs, (int)d, (bf16*)h->ws13);
    interleave_split3_kernel<<<grid_1d(E * hh * l, TPB), TPB, 0, st>>>((const float*)w->w1, (const float*)w->w3,
                                                                       nullptr, (int)E, (int)hh, (int)l,
                                                                       (bf16*)h->w13);
    split3_kernel<<<grid_1d(E * l * hh, TPB), TPB, 0, st>>>((const float*)w->w2, nullptr, (int)(E * l), (int)hh,
                                                            (bf16*)h->w2, (int)(3 * hh), 0);
    split3_kernel<<<grid_1d(d * l, TPB), TPB, 0, st>>>((const float*)w->w_up, nullptr, (int)d, (int)l, (bf16*)h->wy,
                                                       (int)(3 * (l + hs)), 0);
    if (hs)
      split3_kernel<<<grid_1d(d * hs, TPB), TPB, 0, st>>>((const float*)w->ws2, nullptr, (int)d, (int)hs,
                                                          (bf16*)h->wy, (int)(3 * (l + hs)), (int)(3 * l));
  }
  {  // W_comb = W_r (W_down g) in fp64, for the exact decision of ambiguous top-k choices
    const dim3 grid((unsigned)((d + 255) / 256), (unsigned)E);
    if (h->bf)
      combine_router_kernel<bf16><<<grid, 256, 0, st>>>(w->w_router, (const bf16*)w->w_down,
                                                        h->unit_gain ? nullptr : (const bf16*)w->rms_gain, (int)l,
                                                        (int)d, h->wc);
    else
      combine_router_kernel<float><<<grid, 256, 0, st>>>(w->w_router, (const float*)w->w_down,
                                                         (const float*)w->rms_gain, (int)l, (int)d, h->wc);
  }
  CK(cudaGetLastError());
  CK(cudaMemsetAsync(h->c, 0, (size_t)h->E_pad * 4, st));
  if (w->router_bias) CK(cudaMemcpyAsync(h->c, w->router_bias, E * 4, cudaMemcpyDeviceToDevice, st));
  return LMOE_OK;
}

bool gain_is_unit(const lmoe_config& c, const void* g) {
  if (!g) return true;
  const size_t es = c.dtype == LMOE_BF16 ? 2 : 4;
  std::vector<uint8_t> buf(c.d * es);
  if (cudaMemcpy(buf.data(), g, buf.size(), cudaMemcpyDeviceToHost) != cudaSuccess) return false;
  for (int j = 0; j < c.d; ++j) {
    if (es == 2) {
      uint16_t v;
      memcpy(&v, &buf[j * 2], 2);
      if (v != 0x3F80) return false;
    } else {
      float v;
      memcpy(&v, &buf[j * 4], 4);
      if (v != 1.0f) return false;
    }
  }
  return true;
}

// Runs `body(stream)` through the handle's graph cache.  The first call with a new argument key
// runs eagerly on the caller's stream; a repeat of the same key is captured once on the handle's
// private stream into an executable graph, which every later repeat replays on the caller's
// stream.  Eager whenever profiling is on or the caller's stream is itself being captured.
template <typename F>
int run_cached(lmoe_handle* h, GraphCache& g, const void* x, void* y, int T, uint32_t flags, float beta,
               uint64_t state, cudaStream_t st, F body) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (h->profiling || cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
    return body(st);
  }
  if (!g.same(x, y, T, flags, beta, state)) g.reset(x, y, T, flags, beta, state);
  if (g.exec) {
    CK(cudaGraphLaunch(g.exec, st));
    h->launches += g.kernels;
    return LMOE_OK;
  }
  if (g.seen == 0) {
    g.seen = 1;
    return body(st);
  }
  const long long before = h->launches;
  cudaGraph_t graph = nullptr;
  CK(cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal));
  int rc = body(h->cap);
  cudaError_t ce = cudaStreamEndCapture(h->cap, &graph);
  if (rc != LMOE_OK || ce != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();
    h->launches = before;
    return rc != LMOE_OK ? rc : LMOE_ECUDA;
  }
  ce = cudaGraphInstantiate(&g.exec, graph, 0);
  cudaGraphDestroy(graph);
  if (ce != cudaSuccess) {
    g.exec = nullptr;
    return LMOE_ECUDA;
  }
  g.kernels = h->launches - before;
  CK(cudaGraphLaunch(g.exec, st));
  return LMOE_OK;
}

// ---------------------------------------------------------------------- layer backward
// Allocates the backward's workspace on first use.
int bwd_alloc(lmoe_handle* h) {
  if (h->bw) return LMOE_OK;
  const lmoe_config& c = h->cfg;
  const size_t Tm = c.max_tokens, d = c.d, l = c.l, E = c.E, hh = c.h, hs = c.hs;
  BwdWork* b = new (std::nothrow) BwdWork();
  if (!b) return LMOE_ENOMEM;
  b->RP = (h->rows_pad + 127) / 128 * 128;
  const size_t RP = (size_t)b->RP;
  Arena a;
  a.add((void**)&b->xh, Tm * d * 2);
  a.add((void**)&b->ps, Tm * 2 * hs * 2);
  a.add((void**)&b->dps, Tm * 2 * hs * 2);
  a.add((void**)&b->dz, Tm * l * 2);
  a.add((void**)&b->pe, RP * 2 * hh * 2);
  a.add((void**)&b->dpe, RP * 2 * hh * 2);
  a.add((void**)&b->d_o, RP * l * 2);
  a.add((void**)&b->dhe, RP * l * 2);
  a.add((void**)&b->dlogit, Tm * E * 2);
  a.add((void**)&b->dh, Tm * l * 2);
  a.add((void**)&b->dlp, RP * 4);
  a.add((void**)&b->dhr, Tm * l * 4);
  a.add((void**)&b->dxh, Tm * d * 4);
  a.add((void**)&b->gpart, (Tm + kRmsRows - 1) / kRmsRows * d * 4);
  if (cudaMalloc(&b->mem, a.off) != cudaSuccess) {
    delete b;
    return LMOE_ENOMEM;
  }
  for (auto& it : a.items) *it.first = (uint8_t*)b->mem + it.second;
  const long long R = b->RP;
  bool ok = true;
  ok &= make_map(&b->pe_out, b->pe, R, 2 * hh, 2 * hh, 128);
  ok &= make_map(&b->dpe_out, b->dpe, R, 2 * hh, 2 * hh, 128);
  ok &= make_map(&b->dpe_k, b->dpe, R, 2 * hh, 2 * hh, 128);
  ok &= make_map(&b->dpe_mn, b->dpe, R, 2 * hh, 2 * hh, 64);
  ok &= make_map(&b->do_k, b->d_o, R, l, l, 128);
  ok &= make_map(&b->do_mn, b->d_o, R, l, l, 64);
  ok &= make_map(&b->dhe_out, b->dhe, R, l, l, 128);
  ok &= make_map(&b->aperm_mn, h->a_perm, h->rows_pad, l, l, 64);
  ok &= make_map(&b->act_mn, h->act, h->rows_pad, hh, hh, 64);
  if (hs) ok &= make_map(&b->ps_out, b->ps, (long long)Tm, 2 * hs, 2 * hs, 128);
  h->bw = b;
  return ok ? LMOE_OK : LMOE_EINVAL;
}

void bwd_free(lmoe_handle* h) {
  if (!h->bw) return;
  cudaFree(h->bw->mem);
  delete h->bw;
  h->bw = nullptr;
}

// A weight gradient G [M, N] (fp32) = A^T B over K rows (both operands MN-major: A stored [K, M],
// B stored [K, N]), on two-CTA 256-row tiles where M allows.  When the output tiles cannot fill the
// GPU, K is cut into ranges whose partial products are added into the zeroed output by TMA
// reductions.
int wgrad_gemm(lmoe_handle* h, TcParams& p, int M, int N, long long K, size_t out_bytes, void* out,
               size_t out2_bytes, void* out2, cudaStream_t st) {
  const bool pair = M >= 256 && N % 128 == 0;
  const int bn = N % 256 == 0 ? 256 : (N % 128 == 0 ? 128 : 64);
  p.a_mn = 1;
  p.b_mn = 1;
  p.M = M;
  p.M_rows = M;
  p.n_tiles = N / bn;
  p.nseg = 1;
  p.seg[0] = KSeg{0, 0, 0, (int)((K + 63) / 64), 0};
  const int units = pair ? h->sms / 2 : h->sms;  // CTAs, or CTA pairs
  const long long base = (long long)(pair ? (M + 255) / 256 : (M + 127) / 128) * p.n_tiles;
  const int nkb = p.seg[0].nkb;
  // K ranges (at least 4 k-blocks each): as many as fill one wave of tiles.  Measured on a B200
  // with L2-resident operands, a second partial wave cost more than the reductions it saved.
  const int S = (int)std::max<long long>(1, std::min<long long>(units / base, std::max(1, nkb / 4)));
  p.k_split = S;
  if (S > 1) {
    CK(cudaMemsetAsync(out, 0, out_bytes, st));
    if (out2) CK(cudaMemsetAsync(out2, 0, out2_bytes, st));
  }
  const long long tiles = base * S;
  if (pair)
    CK(launch_tc_pair(p, EPI_F32, bn, 2 * (int)std::min<long long>(tiles, units), st));
  else
    CK(launch_tc(p, EPI_F32, bn, (int)std::min<long long>(tiles, units), st));
  h->launches += 1;
  return LMOE_OK;
}

// A dense product of T rows (fp32 or bf16 out) on two-CTA 256-row tiles where T and N allow, else
// on 128-row tiles.  The caller sets the operands, segments and output; this picks the tile width
// and the grid.
int dense_gemm(lmoe_handle* h, TcParams& p, int epi, int T, int N, cudaStream_t st) {
  p.M = T;
  p.M_rows = T;
  const int pbn = (T >= 256 * 8 && epi != EPI_SWIGLU && epi != EPI_SWIGLU3 && epi != EPI_ROUTER && epi != EPI_DOWN3)
                      ? pick_pair_bn(T, N, h->sms)
                      : 0;
  if (pbn) {
    p.n_tiles = N / pbn;
    const long long tiles = (long long)((T + 255) / 256) * p.n_tiles;
    CK(launch_tc_pair(p, epi, pbn, 2 * (int)std::min<long long>(tiles, h->sms / 2), st));
  } else {
    const int bn = pick_bn_for(T, N, h->sms, 64);
    p.n_tiles = N / bn;
    const long long tiles = (long long)((T + 127) / 128) * p.n_tiles;
    CK(launch_tc(p, epi, bn, (int)std::min<long long>(tiles, h->sms), st));
  }
  h->launches += 1;
  return LMOE_OK;
}

// The backward of a bf16 layer with bf16 experts, right after the forward of the same x on the
// same stream (the forward's routing, gathered rows, activations and expert outputs are still in
// the workspace).  Operands are bf16 (the gradients flowing back are rounded to bf16 before each
// product), accumulation fp32; every gradient is written in fp32.
int backward_bf16(lmoe_handle* h, const lmoe_weights* w, const void* x, const void* dy, int T, const lmoe_grads* g,
                  cudaStream_t st) {
  const lmoe_config& c = h->cfg;
  BwdWork* b = h->bw;
  const long long d = c.d, l = c.l, E = c.E, hh = c.h, hs = c.hs;
  const int sms = h->sms;
  bool ok = true;
  // per-call maps of the token-row buffers (their row extent is T, so K = T products read zeros
  // past the last token)
  CUtensorMap dy_k, dy_mn, xh_mn, dps_out, dps_k, dps_mn, dz_out, as_mn, z_mn, dlg_k, dlg_mn, hx_mn, dhr_out,
      dh_k, dh_mn, dxh_out;
  ok &= make_map(&dy_k, dy, T, d, d, 128);
  ok &= make_map(&dy_mn, dy, T, d, d, 64);
  ok &= make_map(&xh_mn, b->xh, T, d, d, 64);
  if (hs) {
    ok &= make_map(&dps_out, b->dps, T, 2 * hs, 2 * hs, 128);
    ok &= make_map(&dps_k, b->dps, T, 2 * hs, 2 * hs, 128);
    ok &= make_map(&dps_mn, b->dps, T, 2 * hs, 2 * hs, 64);
    ok &= make_map(&as_mn, h->a_s, T, hs, hs, 64);
  }
  ok &= make_map(&dz_out, b->dz, T, l, l, 128);
  ok &= make_map(&z_mn, h->z, T, l, l, 64);
  ok &= make_map(&dlg_k, b->dlogit, T, E, E, 128);
  ok &= make_map(&dlg_mn, b->dlogit, T, E, E, 64);
  ok &= make_map(&hx_mn, h->hx, T, l, 3 * l, 64);
  ok &= make_map_f32(&dhr_out, b->dhr, T, l, l, 128);
  ok &= make_map(&dh_k, b->dh, T, l, l, 128);
  ok &= make_map(&dh_mn, b->dh, T, l, l, 64);
  ok &= make_map_f32(&dxh_out, b->dxh, T, d, d, 128);
  // the caller's weights, MN-major (rows = the product's K)
  CUtensorMap wup_mn, ws2_mn, ws1_mn, ws3_mn, w2_mn, w1_mn, w3_mn, wd_mn, wr_hi_mn, wr_mid_mn;
  ok &= make_map(&wup_mn, w->w_up, d, l, l, 64);
  if (hs) {
    ok &= make_map(&ws2_mn, w->ws2, d, hs, hs, 64);
    ok &= make_map(&ws1_mn, w->ws1, hs, d, d, 64);
    ok &= make_map(&ws3_mn, w->ws3, hs, d, d, 64);
  }
  ok &= make_map(&w2_mn, w->w2, E * l, hh, hh, 64);
  ok &= make_map(&w1_mn, w->w1, E * hh, l, l, 64);
  ok &= make_map(&w3_mn, w->w3, E * hh, l, l, 64);
  ok &= make_map(&wd_mn, w->w_down, l, d, d, 64);
  // the router weights: the hi and mid bf16 parts of the fp32 values the handle holds
  ok &= make_map(&wr_hi_mn, h->w_r, E, l, 3 * l, 64);
  ok &= make_map(&wr_mid_mn, (const bf16*)h->w_r + l, E, l, 3 * l, 64);
  // gradient outputs (fp32, boxes of 32 columns x 128 rows)
  CUtensorMap gw1, gw3, gw2, gwr, gwd, gws1, gws3, gws2, gwup;
  ok &= make_map_f32(&gw1, g->w1, E * hh, l, l, 128);
  ok &= make_map_f32(&gw3, g->w3, E * hh, l, l, 128);
  ok &= make_map_f32(&gw2, g->w2, E * l, hh, hh, 128);
  ok &= make_map_f32(&gwr, g->w_router, E, l, l, 128);
  ok &= make_map_f32(&gwd, g->w_down, l, d, d, 128);
  ok &= make_map_f32(&gwup, g->w_up, d, l, l, 128);
  if (hs) {
    ok &= make_map_f32(&gws1, g->ws1, hs, d, d, 128);
    ok &= make_map_f32(&gws3, g->ws3, hs, d, d, 128);
    ok &= make_map_f32(&gws2, g->ws2, d, hs, hs, 128);
  }
  if (!ok) return LMOE_EINVAL;

  // x_hat, the operand of the W_down and shared-expert weight gradients
  CK(launch_k(xhat_kernel, dim3(grid_1d((long long)T * d / 8, 256)), dim3(256), 0, st, 1, (const bf16*)x,
              (const bf16*)w->rms_gain, (const float*)h->r, (long long)T, (int)d, b->xh));
  h->launches += 1;
  if (hs) {
    // dL/d act_s = dy Ws2 and through the SwiGLU (pre-activations saved by the forward):
    // [dL/dp1 | dL/dp3] of the shared expert
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = dy_k;
    p.tmB = ws2_mn;
    p.b_mn = 1;
    p.nseg = 1;
    p.seg[0] = KSeg{0, 0, 0, (int)(d / 64), 0};
    p.tmOut = dps_out;
    p.aux = b->ps;
    p.ld_aux = 2 * hs;
    p.split = hs;
    int rc = dense_gemm(h, p, EPI_SWIGLU_BWD, T, (int)hs, st);
    if (rc) return rc;
  }
  {  // dL/dz = dy W_up
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = dy_k;
    p.tmB = wup_mn;
    p.b_mn = 1;
    p.nseg = 1;
    p.seg[0] = KSeg{0, 0, 0, (int)(d / 64), 0};
    p.tmOut = dz_out;
    int rc = dense_gemm(h, p, EPI_BF16, T, (int)l, st);
    if (rc) return rc;
  }
  // combine and gates: dL/do of every pair, dL/dlogit
  CK(launch_k(combine_bwd_kernel, dim3((T + 7) / 8), dim3(256), 0, st, 1, (const bf16*)b->dz, (const bf16*)h->o,
              (const int*)h->prow, (const float*)h->gates, (const int*)h->idx, (const float*)h->s, T, c.k, (int)l,
              (int)E, b->d_o, b->dlogit, b->dlp));
  h->launches += 1;
  {  // routed experts: dL/d act_e = dL/do W2_e, through the SwiGLU (pre-activations saved by the
     // forward): [dL/dp1 | dL/dp3] (zero past each expert's rows)
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = b->do_k;
    p.tmB = w2_mn;
    p.b_mn = 1;
    p.nseg = 1;
    p.seg[0] = KSeg{0, 0, 0, (int)(l / 64), 0};
    p.grouped = 1;
    const int bn5 = hh % 256 == 0 ? 256 : (hh % 128 == 0 ? 128 : 64);
    p.n_tiles = (int)(hh / bn5);
    p.mtile_table = h->mtiles;
    p.num_mtiles = h->num_mtiles;
    p.b_rows_per_group = (int)l;
    p.tmOut = b->dpe_out;
    p.aux = b->pe;
    p.ld_aux = 2 * hh;
    p.split = hh;
    CK(launch_tc(p, EPI_SWIGLU_BWD, bn5, sms, st));
    // dL/dh of each pair = dL/dp1 W1_e + dL/dp3 W3_e
    p = tc_base(h);
    p.tmA[0] = p.tmA[1] = b->dpe_k;
    p.tmB = w1_mn;
    p.tmB2[0] = w3_mn;
    p.b_mn = 1;
    p.nseg = 2;
    p.seg[0] = KSeg{0, 0, 0, (int)(hh / 64), 0};
    p.seg[1] = KSeg{0, (int)hh, 0, (int)(hh / 64), 1};
    p.grouped = 1;
    const int bn6 = l % 256 == 0 ? 256 : (l % 128 == 0 ? 128 : 64);
    p.n_tiles = (int)(l / bn6);
    p.mtile_table = h->mtiles;
    p.num_mtiles = h->num_mtiles;
    p.b_rows_per_group = (int)hh;
    p.tmOut = b->dhe_out;
    CK(launch_tc(p, EPI_BF16, bn6, sms, st));
    h->launches += 2;
  }
  // rows past each expert's last pair, up to its next 64-row boundary: zero in A_perm, act and
  // dL/do, the operands of the expert weight gradients
  CK(launch_k(pad_zero_kernel, dim3((unsigned)E), dim3(256), 0, st, 1, (const int*)h->offsets,
              (const int*)h->pad_delta, (const int*)h->counts, (bf16*)h->a_perm, (int)l, (bf16*)h->act, (int)hh,
              b->d_o, (int)l));
  h->launches += 1;
  {  // dW1_e, dW3_e = [dL/dp1 | dL/dp3]^T A_perm and dW2_e = (dL/do)^T act over each expert's rows
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = b->dpe_mn;
    p.tmB = b->aperm_mn;
    p.a_mn = p.b_mn = 1;
    p.grouped_k = 1;
    p.k_groups = (int)E;
    p.k_first = h->offsets;
    p.k_pad = h->pad_delta;
    p.k_rows = h->counts;
    p.M = (int)(2 * hh);
    p.M_rows = p.M;
    const int bn7 = l % 256 == 0 ? 256 : (l % 128 == 0 ? 128 : 64);
    p.n_tiles = (int)(l / bn7);
    p.nseg = 1;
    p.seg[0] = KSeg{0, 0, 0, 0, 0};
    p.tmOut = gw1;
    p.tmOut2 = gw3;
    p.out_split = (int)hh;
    // four output boxes in flight when the experts average 256 rows or more (4+ k-blocks per tile:
    // the fp32 stream of gradients limits them; wide layer's backward 14.6-15.2 -> 13.9-14.0 ms),
    // two below (mini_replica, 192 rows: the ring stage they cost mattered more, +10 us)
    const int wepi = (long long)T * c.k >= 256LL * E ? EPI_F32_DEEP : EPI_F32;
    CK(launch_tc(p, wepi, bn7, sms, st));
    p.tmA[0] = p.tmA[1] = b->do_mn;
    p.tmB = b->act_mn;
    p.M = (int)l;
    p.M_rows = p.M;
    const int bn8 = hh % 256 == 0 ? 256 : (hh % 128 == 0 ? 128 : 64);
    p.n_tiles = (int)(hh / bn8);
    p.tmOut = gw2;
    p.out_split = 0;
    CK(launch_tc(p, wepi, bn8, sms, st));
    h->launches += 2;
  }
  // router: dL/dc, dW_r = dlogit^T h, and its part of dL/dh = dlogit W_r
  CK(launch_k(bias_grad_kernel, dim3((unsigned)((E + 7) / 8)), dim3(256), 0, st, 1, (const int*)h->offsets,
              (const int*)h->pad_delta, (const int*)h->counts, (const float*)b->dlp, (int)E, g->router_bias));
  h->launches += 1;
  {
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = dlg_mn;
    p.tmB = hx_mn;
    p.tmOut = gwr;
    int rc = wgrad_gemm(h, p, (int)E, (int)l, T, (size_t)E * l * 4, g->w_router, 0, nullptr, st);
    if (rc) return rc;
    p = tc_base(h);
    p.tmA[0] = p.tmA[1] = dlg_k;
    p.tmB = wr_hi_mn;
    p.tmB2[0] = wr_mid_mn;
    p.b_mn = 1;
    p.nseg = 2;
    p.seg[0] = KSeg{0, 0, 0, (int)(E / 64), 0};
    p.seg[1] = KSeg{0, 0, 0, (int)(E / 64), 1};
    p.tmOut = dhr_out;
    rc = dense_gemm(h, p, EPI_F32, T, (int)l, st);
    if (rc) return rc;
  }
  // dL/dh = the router's part + the experts' parts of the token's pairs
  CK(launch_k(scatter_dh_kernel, dim3((T + 7) / 8), dim3(256), 0, st, 1, (const float*)b->dhr, (const bf16*)b->dhe,
              (const int*)h->prow, T, c.k, (int)l, b->dh));
  h->launches += 1;
  {  // dW_down = (dL/dh)^T x_hat
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = dh_mn;
    p.tmB = xh_mn;
    p.tmOut = gwd;
    int rc = wgrad_gemm(h, p, (int)l, (int)d, T, (size_t)l * d * 4, g->w_down, 0, nullptr, st);
    if (rc) return rc;
  }
  {  // dL/dx_hat = dL/dh W_down + dL/dp1_s Ws1 + dL/dp3_s Ws3
    TcParams p = tc_base(h);
    p.tmA[0] = dh_k;
    p.tmA[1] = hs ? dps_k : dh_k;
    p.tmB = wd_mn;
    if (hs) {
      p.tmB2[0] = ws1_mn;
      p.tmB2[1] = ws3_mn;
    }
    p.b_mn = 1;
    p.nseg = hs ? 3 : 1;
    p.seg[0] = KSeg{0, 0, 0, (int)(l / 64), 0};
    p.seg[1] = KSeg{1, 0, 0, (int)(hs / 64), 1};
    p.seg[2] = KSeg{1, (int)hs, 0, (int)(hs / 64), 2};
    p.tmOut = dxh_out;
    int rc = dense_gemm(h, p, EPI_F32, T, (int)d, st);
    if (rc) return rc;
  }
  if (hs) {  // dWs1, dWs3 = [dL/dp1_s | dL/dp3_s]^T x_hat;  dWs2 = dy^T act_s
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = dps_mn;
    p.tmB = xh_mn;
    p.tmOut = gws1;
    p.tmOut2 = gws3;
    p.out_split = (int)hs;
    int rc = wgrad_gemm(h, p, (int)(2 * hs), (int)d, T, (size_t)hs * d * 4, g->ws1, (size_t)hs * d * 4, g->ws3, st);
    if (rc) return rc;
    p = tc_base(h);
    p.tmA[0] = p.tmA[1] = dy_mn;
    p.tmB = as_mn;
    p.tmOut = gws2;
    rc = wgrad_gemm(h, p, (int)d, (int)hs, T, (size_t)d * hs * 4, g->ws2, 0, nullptr, st);
    if (rc) return rc;
  }
  {  // dW_up = dy^T z
    TcParams p = tc_base(h);
    p.tmA[0] = p.tmA[1] = dy_mn;
    p.tmB = z_mn;
    p.tmOut = gwup;
    int rc = wgrad_gemm(h, p, (int)d, (int)l, T, (size_t)d * l * 4, g->w_up, 0, nullptr, st);
    if (rc) return rc;
  }
  // RMSNorm: dL/dx and dL/dgain
  const int nrb = (T + kRmsRows - 1) / kRmsRows;
  CK(launch_k(rms_bwd_kernel, dim3(nrb), dim3(256), 0, st, 1, (const bf16*)x, (const bf16*)w->rms_gain,
              (const float*)h->r, (const float*)b->dxh, T, (int)d, g->dx, b->gpart));
  if (g->rms_gain)
    CK(launch_k(colsum_kernel, dim3((unsigned)((d + 31) / 32)), dim3(256), 0, st, 1, (const float*)b->gpart, nrb,
                (int)d, g->rms_gain));
  h->launches += 2;
  return LMOE_OK;
}

}  // namespace

// ======================================================================= C ABI
extern "C" {

const char* lmoe_strerror(int code) {
  switch (code) {
    case LMOE_OK: return "ok";
    case LMOE_EINVAL: return "invalid argument";
    case LMOE_ENOMEM: return "out of device memory";
    case LMOE_ECUDA: return "CUDA error";
    case LMOE_EUNSUPPORTED: return "unsupported shape";
    case LMOE_EDEVICE: return "device is not sm_100";
    default: return "unknown error";
  }
}

static void size_handle(lmoe_handle* h, const lmoe_config* cfg) {
  h->cfg = *cfg;
  h->bf = cfg->dtype == LMOE_BF16;
  h->es = h->bf ? 2 : 4;
  h->nblk_max = (cfg->max_tokens + kTokBlock - 1) / kTokBlock;
  h->max_mtiles = (int)(((long long)cfg->max_tokens * cfg->k + kTileRows - 1) / kTileRows) + cfg->E;
  h->ld_bins = (cfg->max_tokens + 31) / 32 * 32;
  h->rows_pad = (long long)cfg->max_tokens * cfg->k + (long long)kTileRows * cfg->E;
  h->q8 = cfg->experts == LMOE_EXPERTS_MXFP8;
  h->E_pad = h->bf ? cfg->E : (cfg->E + 63) / 64 * 64;
}

int lmoe_workspace_bytes(const lmoe_config* cfg, size_t* bytes) {
  int rc = validate(cfg);
  if (rc) return rc;
  if (!bytes) return LMOE_EINVAL;
  lmoe_handle h;
  size_handle(&h, cfg);
  h.unit_gain = false;  // upper bound
  Arena a;
  plan_layout(&h, a);
  *bytes = a.off;
  return LMOE_OK;
}

int lmoe_create(const lmoe_config* cfg, const lmoe_weights* w, void* stream, lmoe_handle** out) {
  if (!out) return LMOE_EINVAL;
  *out = nullptr;
  int rc = validate(cfg);
  if (rc) return rc;
  if (!w || !w->w_down || !w->w_router || !w->w1 || !w->w3 || !w->w2 || !w->w_up) return LMOE_EINVAL;
  if (cfg->hs && (!w->ws1 || !w->ws3 || !w->ws2)) return LMOE_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LMOE_ECUDA;
  int major = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10) return LMOE_EDEVICE;
  lmoe_handle* h = new (std::nothrow) lmoe_handle();
  if (!h) return LMOE_ENOMEM;
  size_handle(h, cfg);
  h->device = dev;
  h->sms = sms;
  h->unit_gain = gain_is_unit(*cfg, w->rms_gain);
  // near-tie width for the exact decision: 2.5 times the bound on the scores' fp32 error (2e-6 at
  // d = 1024, growing like the square root of the longer accumulation: d, or the router's six
  // products over l), so two scores that each err by up to the bound cannot swap unnoticed
  h->tau = 5e-6f * (float)std::max(1.0, std::sqrt(std::max((double)cfg->d, 6.0 * cfg->l) / 1024.0));
  Arena a;
  plan_layout(h, a);
  if (cudaMalloc(&h->arena, a.off) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return LMOE_ENOMEM;
  }
  h->arena_bytes = a.off;
  for (auto& it : a.items) *it.first = h->arena + it.second;
  cudaStream_t st = (cudaStream_t)stream;
  rc = repack(h, w, st);
  if (!rc && cudaMemsetAsync(h->bias, 0, cfg->E * 4, st) != cudaSuccess) rc = LMOE_ECUDA;
  if (!rc && cudaMemsetAsync(h->hist, 0, (size_t)cfg->E * LMOE_NBINS * 4, st) != cudaSuccess) rc = LMOE_ECUDA;
  if (!rc && cudaMemsetAsync(h->ntok, 0, 8, st) != cudaSuccess) rc = LMOE_ECUDA;
  if (!rc && cudaMemsetAsync(h->load, 0, (size_t)cfg->E * 8, st) != cudaSuccess) rc = LMOE_ECUDA;
  if (!rc && cudaMemsetAsync(h->status, 0, 4, st) != cudaSuccess) rc = LMOE_ECUDA;
  if (!rc && cudaMemsetAsync(h->qb_done, 0, 4, st) != cudaSuccess) rc = LMOE_ECUDA;
  if (!rc) rc = h->bf ? build_maps(h) : build_maps_f32(h);
  if (!rc && cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking) != cudaSuccess) rc = LMOE_ECUDA;
  if (!rc && cudaStreamCreateWithFlags(&h->cp_in, cudaStreamNonBlocking) != cudaSuccess) rc = LMOE_ECUDA;
  if (!rc && cudaStreamCreateWithFlags(&h->cp_out, cudaStreamNonBlocking) != cudaSuccess) rc = LMOE_ECUDA;
  if (!rc && cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) != cudaSuccess) rc = LMOE_ECUDA;
  if (!rc && (cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
              cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess))
    rc = LMOE_ECUDA;
  for (int i = 0; !rc && i < 2; ++i)
    if (cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->ev_fwd[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming) != cudaSuccess)
      rc = LMOE_ECUDA;
  if (rc) {
    cudaStreamSynchronize(st);
    cudaFree(h->arena);
    delete h;
    return rc;
  }
  *out = h;
  return LMOE_OK;
}

int lmoe_destroy(lmoe_handle* h) {
  if (!h) return LMOE_EINVAL;
  cudaDeviceSynchronize();
  bwd_free(h);
  for (auto& r : h->prof)
    for (auto& e : r.ev) cudaEventDestroy(e);
  for (auto& g : h->g_fwd) g.reset(nullptr, nullptr, -1, 0, 0.f, 0);
  h->g_qb.reset(nullptr, nullptr, -1, 0, 0.f, 0);
  h->g_bwd.reset(nullptr, nullptr, -1, 0, 0.f, 0);
  if (h->cap) cudaStreamDestroy(h->cap);
  if (h->cp_in) cudaStreamDestroy(h->cp_in);
  if (h->cp_out) cudaStreamDestroy(h->cp_out);
  if (h->side) cudaStreamDestroy(h->side);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  for (int i = 0; i < 2; ++i) {
    if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
    if (h->ev_fwd[i]) cudaEventDestroy(h->ev_fwd[i]);
    if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
  }
  cudaFree(h->arena);
  delete h;
  return LMOE_OK;
}

// Forward of lmoe_forward; save_pre (a training step) also stores the SwiGLU pre-activations for
// the backward (a separate graph: its key carries kSavePre).
constexpr uint32_t kSavePre = 1u << 15;
static int forward_impl(lmoe_handle* h, const void* x, void* y, int32_t T, uint32_t flags, bool save_pre,
                        void* stream);

int lmoe_forward(lmoe_handle* h, const void* x, void* y, int32_t T, uint32_t flags, void* stream) {
  return forward_impl(h, x, y, T, flags & ~kSavePre, false, stream);
}

static int forward_impl(lmoe_handle* h, const void* x, void* y, int32_t T, uint32_t flags, bool save_pre,
                        void* stream) {
  if (!h || T < 0 || T > h->cfg.max_tokens) return LMOE_EINVAL;
  if (T == 0) return LMOE_OK;
  if (!x || !y || ((uintptr_t)x & 15) || ((uintptr_t)y & 15)) return LMOE_EINVAL;
  const size_t bytes = (size_t)T * h->cfg.d * h->es;
  if ((const char*)x < (const char*)y + bytes && (const char*)y < (const char*)x + bytes) return LMOE_EINVAL;
  cudaStream_t st = (cudaStream_t)stream;
  h->last_T = T;
  flags &= ~LMOE_ASYNC_OUTPUT;  // a host-buffer option only
  const bool upd = (flags & LMOE_UPDATE_BIAS) != 0;
  if (upd && (!(flags & LMOE_RECORD_STATS) || !h->upd_set)) return LMOE_EINVAL;
  const StatsState pre = h->ss;
  // graph key: the arguments, the update's step and flags, the statistics state
  const uint32_t kflags = flags | (upd ? h->upd_flags << 16 : 0u) | (save_pre ? kSavePre : 0u);
  const float kbeta = upd ? h->upd_beta : 0.f;
  // the cached graph of these arguments, else the least recently used one
  int gi = h->g_fwd[0].same(x, y, T, kflags, kbeta, pre.key()) ? 0
           : h->g_fwd[1].same(x, y, T, kflags, kbeta, pre.key()) ? 1
           : (h->g_used[0] <= h->g_used[1] ? 0 : 1);
  h->g_used[gi] = ++h->g_tick;
  int rc = run_cached(h, h->g_fwd[gi], x, y, T, kflags, kbeta, pre.key(), st, [&](cudaStream_t s) {
    prof_open(h, ST_RMS, ST_UP - ST_RMS + 1);
    int r = h->bf ? forward_bf16(h, x, y, T, flags, pre, s, save_pre) : forward_f32(h, x, y, T, flags, pre, s);
    prof_close(h, s);
    if (!r && upd && h->profiling) {  // profiled: the update after the forward, timed as its own stage
      prof_open(h, ST_QB_UPDATE, 1);
      mark(h, ST_QB_UPDATE, s);
      r = launch_qb(h, h->upd_beta, h->upd_flags, after_routing(pre, T, flags), s);
      prof_close(h, s);
    }
    return r;
  });
  if (rc == LMOE_OK) {
    h->ss = after_routing(pre, T, flags);
    if (upd) {  // the update consumed every statistic recorded so far
      h->ss.pend_T = 0;
      h->ss.hist_live = false;
    }
  }
  return rc;
}

int lmoe_forward_backward(lmoe_handle* h, const lmoe_weights* w, const void* x, const void* dy, void* y, int32_t T,
                          uint32_t flags, const lmoe_grads* g, void* stream) {
  if (!h || !w || !g || T < 0 || T > h->cfg.max_tokens) return LMOE_EINVAL;
  if (!h->bf || h->q8) return LMOE_EUNSUPPORTED;
  if (flags & (LMOE_UPDATE_BIAS | LMOE_ASYNC_OUTPUT)) return LMOE_EINVAL;
  const lmoe_config& c = h->cfg;
  // 128-row tiles of the weight gradients never straddle two experts or the W1 / W3 (Ws1 / Ws3)
  // boundary
  if (c.l % 128 || c.h % 128 || c.hs % 128) return LMOE_EUNSUPPORTED;
  if (!w->w_down || !w->w_router || !w->w1 || !w->w3 || !w->w2 || !w->w_up) return LMOE_EINVAL;
  if (c.hs && (!w->ws1 || !w->ws3 || !w->ws2)) return LMOE_EINVAL;
  if (!g->dx || !g->w_down || !g->w_router || !g->router_bias || !g->w1 || !g->w3 || !g->w2 || !g->w_up)
    return LMOE_EINVAL;
  if (c.hs && (!g->ws1 || !g->ws3 || !g->ws2)) return LMOE_EINVAL;
  if (!dy || ((uintptr_t)dy & 15)) return LMOE_EINVAL;
  if (T == 0) return LMOE_OK;
  int rc = bwd_alloc(h);
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  rc = forward_impl(h, x, y, T, flags, true, stream);
  if (rc) return rc;
  // the backward is cached as a graph of its own (its host work, 40-odd tensor maps and 25-odd
  // launches, is then one replay): its key is x, dy, T and every pointer of w and g, since the
  // captured tensor maps and kernel arguments hold them
  const void* ptrs[23] = {w->rms_gain, w->w_down, w->w_router, w->router_bias, w->w1, w->w3, w->w2, w->w_up,
                          w->ws1, w->ws3, w->ws2, g->dx, g->rms_gain, g->w_down, g->w_router, g->router_bias,
                          g->w1, g->w3, g->w2, g->w_up, g->ws1, g->ws3, g->ws2};
  static_assert(sizeof ptrs == sizeof h->bwd_ptrs, "backward graph key");
  if (memcmp(ptrs, h->bwd_ptrs, sizeof ptrs) != 0) {
    memcpy(h->bwd_ptrs, ptrs, sizeof ptrs);
    h->g_bwd.reset(nullptr, nullptr, -1, 0, 0.f, 0);
  }
  return run_cached(h, h->g_bwd, x, const_cast<void*>(dy), T, 0, 0.f, 0, st,
                    [&](cudaStream_t s) { return backward_bf16(h, w, x, dy, T, g, s); });
}

int lmoe_forward_host(lmoe_handle* h, const void* x_host, void* y_host, int32_t T, uint32_t flags, void* stream) {
  if (!h || !x_host || !y_host || T < 0 || T > h->cfg.max_tokens) return LMOE_EINVAL;
  if (T == 0) return LMOE_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t bytes = (size_t)T * h->cfg.d * h->es;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
    // under the caller's stream capture everything stays on its stream (an output copy still in
    // flight on the handle's own stream would race with this forward's output)
    if (h->out_pending[0] || h->out_pending[1]) return LMOE_EINVAL;
    CK(cudaMemcpyAsync(h->x_stage, x_host, bytes, cudaMemcpyHostToDevice, st));
    int rc = lmoe_forward(h, h->x_stage, h->y_stage, T, flags & ~LMOE_ASYNC_OUTPUT, stream);
    if (rc) return rc;
    CK(cudaMemcpyAsync(y_host, h->y_stage, bytes, cudaMemcpyDeviceToHost, st));
    return LMOE_OK;
  }
  // the input copy runs on the handle's copy stream into the staging buffer this call owns, once
  // the forward that last read that buffer has finished; the forward waits for the copy (and for
  // an output copy still reading this slot's output buffer)
  const int sl = h->host_slot;
  void* xs = sl ? h->x_stage2 : h->x_stage;
  void* ys = sl ? h->y_stage2 : h->y_stage;
  if (h->fwd_recorded[sl]) CK(cudaStreamWaitEvent(h->cp_in, h->ev_fwd[sl], 0));
  CK(cudaMemcpyAsync(xs, x_host, bytes, cudaMemcpyHostToDevice, h->cp_in));
  CK(cudaEventRecord(h->ev_in[sl], h->cp_in));
  CK(cudaStreamWaitEvent(st, h->ev_in[sl], 0));
  if (h->out_pending[sl]) {
    CK(cudaStreamWaitEvent(st, h->ev_out[sl], 0));
    h->out_pending[sl] = false;
  }
  int rc = lmoe_forward(h, xs, ys, T, flags & ~LMOE_ASYNC_OUTPUT, stream);
  if (rc) return rc;
  CK(cudaEventRecord(h->ev_fwd[sl], st));
  h->fwd_recorded[sl] = true;
  h->host_slot ^= 1;
  if (flags & LMOE_ASYNC_OUTPUT) {
    // the output copy leaves `stream`: the next call's forward overlaps it
    CK(cudaStreamWaitEvent(h->cp_out, h->ev_fwd[sl], 0));
    CK(cudaMemcpyAsync(y_host, ys, bytes, cudaMemcpyDeviceToHost, h->cp_out));
    CK(cudaEventRecord(h->ev_out[sl], h->cp_out));
    h->out_pending[sl] = true;
    h->last_out = sl;
  } else {
    CK(cudaMemcpyAsync(y_host, ys, bytes, cudaMemcpyDeviceToHost, st));
  }
  return LMOE_OK;
}

int lmoe_host_wait(lmoe_handle* h, void* stream) {
  if (!h) return LMOE_EINVAL;
  // cp_out runs its copies in order, so the last one's event covers every earlier one
  if (h->last_out >= 0) CK(cudaStreamWaitEvent((cudaStream_t)stream, h->ev_out[h->last_out], 0));
  return LMOE_OK;
}

int lmoe_route_scores(lmoe_handle* h, const float* scores, int32_t T, uint32_t flags, void* stream) {
  if (!h || !scores || T < 0 || T > h->cfg.max_tokens) return LMOE_EINVAL;
  if (T == 0) return LMOE_OK;
  cudaStream_t st = (cudaStream_t)stream;
  CK(cudaMemcpyAsync(h->s, scores, (size_t)T * h->cfg.E * 4, cudaMemcpyDeviceToDevice, st));
  prof_open(h, ST_TOPK, ST_HIST - ST_TOPK + 1);
  const StatsState pre = h->ss;
  flags &= LMOE_RECORD_STATS;  // the routing stage alone runs no update
  int rc = route_from_scores(h, T, flags, pre, nullptr, st);
  prof_close(h, st);
  if (rc == LMOE_OK) h->ss = after_routing(pre, T, flags);
  return rc;
}

int lmoe_qb_update(lmoe_handle* h, float beta, uint32_t flags, void* stream) {
  if (!h || !(beta == beta)) return LMOE_EINVAL;
  if ((flags & LMOE_QB_LITERAL) && (flags & LMOE_BIAS_SIGN)) return LMOE_EINVAL;
  cudaStream_t st = (cudaStream_t)stream;
  const StatsState pre = h->ss;
  int rc = run_cached(h, h->g_qb, nullptr, nullptr, 0, flags, beta, pre.key(), st, [&](cudaStream_t s) {
    prof_open(h, ST_QB_UPDATE, 1);
    mark(h, ST_QB_UPDATE, s);
    int r = launch_qb(h, beta, flags, pre, s);
    prof_close(h, s);
    return r;
  });
  if (rc == LMOE_OK) {
    h->ss.pend_T = 0;
    h->ss.hist_live = false;
  }
  return rc;
}

int lmoe_set_update(lmoe_handle* h, float beta, uint32_t flags) {
  if (!h || !(beta == beta)) return LMOE_EINVAL;
  if ((flags & LMOE_QB_LITERAL) && (flags & LMOE_BIAS_SIGN)) return LMOE_EINVAL;
  h->upd_beta = beta;
  h->upd_flags = flags & (LMOE_QB_LITERAL | LMOE_BIAS_SIGN);
  h->upd_set = true;
  return LMOE_OK;
}

int lmoe_get_routing(lmoe_handle* h, int32_t* idx, float* gates, float* scores, int32_t* counts, int32_t* offsets,
                     int32_t* perm, int32_t* inv, void* stream) {
  if (!h) return LMOE_EINVAL;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t T = h->last_T, k = h->cfg.k, E = h->cfg.E;
  auto cp = [&](void* dst, const void* src, size_t bytes) {
    return dst && bytes ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) : cudaSuccess;
  };
  CK(cp(idx, h->idx, T * k * 4));
  CK(cp(gates, h->gates, T * k * 4));
  CK(cp(scores, h->s, T * E * 4));
  CK(cp(counts, h->counts, E * 4));
  CK(cp(offsets, h->offsets, (E + 1) * 4));
  CK(cp(perm, h->perm, T * k * 4));
  CK(cp(inv, h->inv, T * k * 4));
  return LMOE_OK;
}

int lmoe_get_bias(lmoe_handle* h, float* b, void* stream) {
  if (!h || !b) return LMOE_EINVAL;
  CK(cudaMemcpyAsync(b, h->bias, h->cfg.E * 4, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return LMOE_OK;
}

int lmoe_set_bias(lmoe_handle* h, const float* b, void* stream) {
  if (!h || !b) return LMOE_EINVAL;
  CK(cudaMemcpyAsync(h->bias, b, h->cfg.E * 4, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return LMOE_OK;
}

int lmoe_get_hist(lmoe_handle* h, uint32_t* hist, int64_t* ntok, void* stream) {
  if (!h) return LMOE_EINVAL;
  cudaStream_t st = (cudaStream_t)stream;
  if (h->ss.pend_T) {  // count the pending bins into the accumulated histogram first
    int rc = flush_bins(h, h->ss.pend_T, h->ss.pend_buf, st);
    if (rc) return rc;
    h->ss.pend_T = 0;
    h->ss.hist_live = true;
  }
  if (hist) CK(cudaMemcpyAsync(hist, h->hist, (size_t)h->cfg.E * LMOE_NBINS * 4, cudaMemcpyDeviceToDevice, st));
  if (ntok) CK(cudaMemcpyAsync(ntok, h->ntok, 8, cudaMemcpyDeviceToDevice, st));
  return LMOE_OK;
}

int lmoe_set_hist(lmoe_handle* h, const uint32_t* hist, const int64_t* ntok, void* stream) {
  if (!h || !hist || !ntok) return LMOE_EINVAL;
  cudaStream_t st = (cudaStream_t)stream;
  CK(cudaMemcpyAsync(h->hist, hist, (size_t)h->cfg.E * LMOE_NBINS * 4, cudaMemcpyDeviceToDevice, st));
  CK(cudaMemcpyAsync(h->ntok, ntok, 8, cudaMemcpyDeviceToDevice, st));
  h->ss.pend_T = 0;  // the given statistics replace everything recorded so far
  h->ss.hist_live = true;
  return LMOE_OK;
}

int lmoe_get_load(lmoe_handle* h, int64_t* load, void* stream) {
  if (!h || !load) return LMOE_EINVAL;
  CK(cudaMemcpyAsync(load, h->load, (size_t)h->cfg.E * 8, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return LMOE_OK;
}

int lmoe_set_load(lmoe_handle* h, const int64_t* load, void* stream) {
  if (!h || !load) return LMOE_EINVAL;
  CK(cudaMemcpyAsync(h->load, load, (size_t)h->cfg.E * 8, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return LMOE_OK;
}

int lmoe_get_status(lmoe_handle* h, uint32_t* status) {
  if (!h || !status) return LMOE_EINVAL;
  CK(cudaDeviceSynchronize());
  CK(cudaMemcpy(status, h->status, 4, cudaMemcpyDeviceToHost));
  CK(cudaMemset(h->status, 0, 4));
  return LMOE_OK;
}

int lmoe_profile_enable(lmoe_handle* h, int32_t enable) {
  if (!h) return LMOE_EINVAL;
  h->profiling = enable != 0;
  return LMOE_OK;
}

int lmoe_profile_read(lmoe_handle* h, float* ms, int32_t n, int32_t* calls) {
  if (!h || !ms || n < ST_COUNT) return LMOE_EINVAL;
  CK(cudaDeviceSynchronize());
  for (int i = 0; i < ST_COUNT; ++i) ms[i] = 0.f;
  int forwards = 0;
  for (int r = 0; r < h->prof_used; ++r) {
    const ProfRecord& pr = h->prof[r];
    if (pr.first == ST_RMS) ++forwards;
    for (int i = 0; i < pr.n; ++i) {
      float t = 0.f;
      if (cudaEventElapsedTime(&t, pr.ev[i], pr.ev[i + 1]) == cudaSuccess) ms[pr.first + i] += t;
    }
  }
  if (calls) *calls = forwards;
  h->prof_used = 0;
  cudaGetLastError();
  return LMOE_OK;
}

const char* lmoe_stage_name(int32_t i) { return (i >= 0 && i < ST_COUNT) ? kStageNames[i] : nullptr; }

int lmoe_launch_count(lmoe_handle* h, int64_t* n) {
  if (!h || !n) return LMOE_EINVAL;
  *n = h->launches;
  return LMOE_OK;
}

int lmoe_gemm_bf16(const void* a, const void* b, float* c, int32_t M, int32_t N, int32_t K, void* stream) {
  if (!a || !b || !c || M <= 0 || N <= 0 || K <= 0 || N % 64 || K % 64) return LMOE_EINVAL;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int bn = pick_bn(N);
  const bool pair = M >= 256 && bn >= 128;  // the two-CTA variant, so tests exercise it
  TcParams p;
  memset(&p, 0, sizeof(p));
  if (!make_map(&p.tmA[0], a, M, K, K, 128) || !make_map(&p.tmB, b, N, K, K, pair ? bn / 2 : bn)) return LMOE_EINVAL;
  p.tmA[1] = p.tmA[0];
  p.nseg = 1;
  p.seg[0] = {0, 0, 0, K / 64};
  p.M = M;
  p.M_rows = M;
  p.n_tiles = N / bn;
  if (!make_map_f32(&p.tmOut, c, M, N, N, 128)) return LMOE_EINVAL;
  if (pair) {
    const int tiles = ((M + 255) / 256) * p.n_tiles;
    CK(launch_tc_pair(p, EPI_F32, bn, 2 * (tiles < sms / 2 ? tiles : sms / 2), (cudaStream_t)stream));
  } else {
    const int tiles = ((M + 127) / 128) * p.n_tiles;
    CK(launch_tc(p, EPI_F32, bn, tiles < sms ? tiles : sms, (cudaStream_t)stream));
  }
  return LMOE_OK;
}

int lmoe_gemm_bf16_ex(const void* a, int32_t a_mn, const void* b, int32_t b_mn, float* c, int32_t M, int32_t N,
                      int32_t K, int32_t k_split, void* stream) {
  if (!a || !b || !c || M <= 0 || N <= 0 || K <= 0 || N % 64 || K % 8 || k_split < 1) return LMOE_EINVAL;
  if ((a_mn && M % 8) || (b_mn && N % 8)) return LMOE_EINVAL;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int bn = pick_bn(N);
  const bool pair = M >= 256 && bn >= 128;  // the two-CTA variant, so tests exercise it
  TcParams p;
  memset(&p, 0, sizeof(p));
  bool ok = a_mn ? make_map(&p.tmA[0], a, K, M, M, 64) : make_map(&p.tmA[0], a, M, K, K, 128);
  ok &= b_mn ? make_map(&p.tmB, b, K, N, N, 64) : make_map(&p.tmB, b, N, K, K, pair ? bn / 2 : bn);
  ok &= make_map_f32(&p.tmOut, c, M, N, N, 128);
  if (!ok) return LMOE_EINVAL;
  p.tmA[1] = p.tmA[0];
  p.a_mn = a_mn ? 1 : 0;
  p.b_mn = b_mn ? 1 : 0;
  p.nseg = 1;
  p.seg[0] = KSeg{0, 0, 0, (K + 63) / 64, 0};
  if (k_split > p.seg[0].nkb) return LMOE_EINVAL;
  p.k_split = k_split;
  p.M = M;
  p.M_rows = M;
  p.n_tiles = N / bn;
  cudaStream_t st = (cudaStream_t)stream;
  if (k_split > 1) CK(cudaMemsetAsync(c, 0, (size_t)M * N * 4, st));
  if (pair) {
    const long long tiles = (long long)((M + 255) / 256) * p.n_tiles * k_split;
    CK(launch_tc_pair(p, EPI_F32, bn, 2 * (int)(tiles < sms / 2 ? tiles : sms / 2), st));
  } else {
    const long long tiles = (long long)((M + 127) / 128) * p.n_tiles * k_split;
    CK(launch_tc(p, EPI_F32, bn, (int)(tiles < sms ? tiles : sms), st));
  }
  return LMOE_OK;
}

// ---------------------------------------------------------------- routing without allocation
// Scratch of lmoe_route_noalloc: a fixed device array in this library's image.  Every GPU that
// loads the library holds it until the process exits.  Its name is only a host-side stand-in;
// kernels get its device address, taken once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LMOE_NOALLOC_SCRATCH_BYTES];

static size_t noalloc_bytes(long long T, long long E, long long k, size_t* off_rank, size_t* off_cnt,
                            size_t* off_base, size_t* off_tiles, size_t* off_delta, size_t* off_c32,
                            size_t* off_ntiles) {
  const long long nblk = (T + kTokBlock - 1) / kTokBlock;
  const long long mtiles = (T * k + kTileRows - 1) / kTileRows + E;
  size_t o = 0;
  *off_rank = o;
  o += align_up((size_t)(T * k) * 4, 256);
  *off_cnt = o;
  o += align_up((size_t)(nblk * E) * 4, 256);
  *off_base = o;
  o += align_up((size_t)(nblk * E) * 4, 256);
  *off_tiles = o;
  o += align_up((size_t)mtiles * 8, 256);
  *off_delta = o;
  o += align_up((size_t)E * 4, 256);
  *off_c32 = o;
  o += align_up((size_t)kCountCopies * E * 4, 256);
  *off_ntiles = o;
  o += 256;
  return o;
}

int lmoe_route_noalloc(const float* scores, const float* bias, int32_t T, int32_t E, int32_t k, int32_t* idx,
                       float* gates, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                       uint32_t* status, void* stream) {
  if (!scores || !bias || !idx || !gates || !counts || !offsets || !perm || !inv || !status) return LMOE_EINVAL;
  if (T < 0 || E <= 0 || k <= 0 || k > E) return LMOE_EINVAL;
  if (E > 1024 || k > 32) return LMOE_EUNSUPPORTED;  // the same limits as lmoe_create
  size_t o_rank, o_cnt, o_base, o_tiles, o_delta, o_c32, o_ntiles;
  if (noalloc_bytes(T, E, k, &o_rank, &o_cnt, &o_base, &o_tiles, &o_delta, &o_c32, &o_ntiles) >
      LMOE_NOALLOC_SCRATCH_BYTES)
    return LMOE_EUNSUPPORTED;
  // set-up, once per device: the device address of the scratch array
  static std::mutex mu;
  static unsigned char* base_of[64] = {};
  int dev = 0;
  CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return LMOE_EDEVICE;
  unsigned char* base;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!base_of[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return LMOE_ECUDA;
      }
      base_of[dev] = static_cast<unsigned char*>(p);
    }
    base = base_of[dev];
  }
  cudaStream_t st = (cudaStream_t)stream;
  CK(cudaMemsetAsync(status, 0, sizeof(uint32_t), st));  // this call's faults only
  if (T == 0) {
    CK(cudaMemsetAsync(counts, 0, (size_t)E * sizeof(int32_t), st));
    CK(cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * sizeof(int32_t), st));
    return LMOE_OK;
  }
  int* rank = reinterpret_cast<int*>(base + o_rank);
  int* blkcnt = reinterpret_cast<int*>(base + o_cnt);
  int* blkbase = reinterpret_cast<int*>(base + o_base);
  int2* tiles = reinterpret_cast<int2*>(base + o_tiles);
  int* delta = reinterpret_cast<int*>(base + o_delta);
  int* counts32 = reinterpret_cast<int*>(base + o_c32);
  int* ntiles = reinterpret_cast<int*>(base + o_ntiles);
  // every scratch word is written before it is read, except the count copies, which the top-k
  // blocks add into; faults (NaN score, index out of range) go to the caller's status word
  CK(cudaMemsetAsync(counts32, 0, (size_t)kCountCopies * E * sizeof(int), st));
  TopkArgs ta{scores, bias, T, E, k, idx, rank, blkcnt, counts32, gates, nullptr, 0, TopkRefine{}, status};
  CK(launch_topk(ta, st));
  const int nblk = (T + kTokBlock - 1) / kTokBlock;
  plan_kernel<<<(E + kPlanExperts - 1) / kPlanExperts, 1024, 0, st>>>(counts32, counts, blkcnt, nblk, E, offsets, delta, blkbase, tiles,
                                               ntiles, nullptr);
  CK(cudaGetLastError());
  const int pairs = T * k;
  gather_kernel<float><<<(pairs + 8 * kGatherPairs - 1) / (8 * kGatherPairs), 256, 0, st>>>(
      nullptr, 0, 0, idx, rank, blkbase, nullptr, T, E, k, perm, inv, nullptr, nullptr, nullptr, 0, status);
  CK(cudaGetLastError());
  return LMOE_OK;
}

// ---------------------------------------------------------------- failure-detection check
// One thread waits, with the pipelines' bounded wait, on an mbarrier that nothing ever completes.
__global__ void watchdog_selftest_kernel(uint32_t* status, long long limit_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(&bar, 0, &abort_flag, status, limit_cycles)) set_status(status, LMOE_STATUS_WATCHDOG);
  }
}

int lmoe_watchdog_selftest(uint32_t* status_dev, int32_t limit_us, void* stream) {
  if (!status_dev || limit_us <= 0 || limit_us > 2000000) return LMOE_EINVAL;
  // ~2000 SM cycles per microsecond at B200 clocks; the exact bound only has to be finite
  watchdog_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status_dev, (long long)limit_us * 2000);
  CK(cudaGetLastError());
  return LMOE_OK;
}

}  // extern "C"
