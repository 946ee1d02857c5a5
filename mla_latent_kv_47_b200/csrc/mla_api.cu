// mla_api.cu -- the C ABI declared in include/mla.h: argument checks, the
// workspace layout, TMA tensor maps, and the launch sequence of each entry
// point.  Every arithmetic step runs in the kernels of this directory.
#include "mla.h"

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "attn_decode_sh.cuh"
#include "attn_decode_tc.cuh"
#include "attn_prefill_tc.cuh"
#include "gemm_tc.cuh"
#include "simt.cuh"
#include "uv_combine.cuh"

using namespace mla;

namespace {

constexpr int kMaxWorkers = 296;        // attention workers (partial slots beyond B)
constexpr int kMaxGemmCtas = 296;       // split-K target: two CTAs per SM on 148 SMs
constexpr size_t kAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace: [status | split-K partials] followed by ONE of the decode region
// (sized by the batch) or the prefill region (sized by the number of key
// tokens); a call uses only its own region.  Apart from the status word, every
// region is written in full by a kernel of the call before any kernel reads it.
struct Layout {
  size_t status, gpart, base_end;
  size_t tile_start, seg_start, rope, cq, qc, qlat, olat, o, opart, ml, nkv, nq, decode_end;
  size_t p_rope, p_cq, p_qp, p_rows, p_kc, p_v, p_out, p_nkv, p_nq, prefill_end;
};

int elem_size(const mla_dims& d) { return d.dtype == MLA_FP32 ? 4 : 2; }
int row_elems(const mla_dims& d) { return d.d_c + d.d_R; }
bool cache_fp8(const mla_dims& d) { return d.cache_format == MLA_CACHE_E4M3; }
// Bytes of one cache row (the layouts of mla_cache_format).
int row_bytes(const mla_dims& d) {
  return cache_fp8(d) ? d.d_c + 2 * d.d_R + 16 : row_elems(d) * elem_size(d);
}

int pick_bn(int N) { return N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256; }

// gpart_bn: widest split-K tile the call may use; workers: attention workers
// (partial slots beyond the batch).
Layout make_layout_sized(const mla_dims& d, int max_batch, int max_tokens, int gpart_bn, int workers) {
  Layout L{};
  const size_t es = elem_size(d);
  const size_t B = static_cast<size_t>(max_batch < 1 ? 1 : max_batch);
  const size_t T = static_cast<size_t>(max_tokens < 1 ? 1 : max_tokens);
  const size_t nh = d.n_h, dh = d.d_h, row = row_elems(d);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, kAlign); return o; };
  L.status = take(256);
  L.gpart = take(static_cast<size_t>(kMaxGemmCtas) * gpart_bn * 128 * sizeof(float));
  L.base_end = off;
  L.tile_start = take((B + 1) * sizeof(int));
  L.seg_start = take((B + 1) * sizeof(int));
  L.rope = take(B * (d.d_R / 2 + 1) * 2 * sizeof(float));
  L.cq = take(B * (d.d_cq ? d.d_cq : 1) * es);
  L.qc = take(B * nh * dh * es);
  L.qlat = take(B * nh * row * es);
  L.olat = take(B * nh * d.d_c * es);
  L.o = take(B * nh * dh * es);
  L.opart = take((B + workers) * nh * d.d_c * sizeof(float));
  L.ml = take((B + workers) * nh * 2 * sizeof(float));
  L.nkv = take(B * d.d_c * sizeof(float));                      // c^KV before the RMSNorm (with g_kv)
  L.nq = take(B * (d.d_cq ? d.d_cq : 1) * sizeof(float));       // c^Q before the RMSNorm (with g_q)
  L.decode_end = off;
  off = L.base_end;
  L.p_rope = take(T * (d.d_R / 2 + 1) * 2 * sizeof(float));
  L.p_cq = take(T * (d.d_cq ? d.d_cq : 1) * es);
  L.p_qp = take(T * nh * (dh + d.d_R) * es);
  L.p_rows = take(T * row * es);
  L.p_kc = take(T * nh * dh * es);
  L.p_v = take(T * nh * dh * es);
  L.p_out = take(T * nh * dh * es);
  // the latents before the RMSNorm are consumed before K^C and V are formed,
  // so they share those buffers when they fit
  const size_t kv_bytes = T * nh * dh * es;
  L.p_nq = T * d.d_cq * sizeof(float) <= kv_bytes ? L.p_kc : take(T * (d.d_cq ? d.d_cq : 1) * sizeof(float));
  L.p_nkv = T * d.d_c * sizeof(float) <= kv_bytes ? L.p_v : take(T * d.d_c * sizeof(float));
  L.prefill_end = off;
  return L;
}

Layout make_layout(const mla_dims& d, int max_batch, int max_tokens) {
  return make_layout_sized(d, max_batch, max_tokens, 256, kMaxWorkers);
}

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D byte tensor [rows x cols] with row stride `ld` bytes; box {box_cols, box_rows}, no swizzle.
bool make_map_2d_u8(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld, uint32_t box_cols,
                    uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor [rows x cols] with row stride `ld` elements; box {64, box_rows}; 128-byte swizzle.
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ GEMM description
struct GemmSpec {
  int mode = GEMM_DENSE;
  int nseg = 0;
  const void* A[kMaxSeg] = {};
  int rows[kMaxSeg] = {};       // dense: rows of each weight; per-head: output rows per head
  long long a_ld = 0;           // dense/K-major: row stride of A (elements) = K;  MN-major: row stride (d_c)
  long long a_total_rows = 0;   // per-head modes: rows of the whole weight tensor
  int K = 0;
  Epi epi[kMaxSeg] = {};
  const void* X = nullptr;
  long long x_cols = 0, x_ld = 0;
  int N = 0;
  int heads = 1;
  int head_rows = 0;            // rows of A per head
  int b_head_stride = 0;        // X column offset per head
  TokenMap tok{};
  bool x_independent = false;   // X is a call input (h): the GEMM need not wait for the kernel before it
};

struct Ctx {
  mla_dims d;
  Layout L;
  uint8_t* ws;
  int* status;
  cudaStream_t st;
  int num_sms;
  bool pdl = false;  // chain the call's kernels with programmatic dependent launch
};

std::atomic<unsigned long long> g_kernel_launches{0};  // diagnostic: kernels launched by this library

// Launches `kern` on the call's stream; with pdl the kernel may begin while
// its predecessor drains (every kernel here calls griddep_wait() before it
// reads or writes anything an earlier kernel touches).
template <typename... KArgs, typename... Args>
mla_status launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                  Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// launch() with clusters of cz CTAs along grid z (gridDim.z == cz).
template <typename... KArgs, typename... Args>
mla_status launch_cluster_z(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                            int cz, Args... args) {
  if (cz <= 1) return launch(kern, grid, block, smem, st, pdl, args...);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = cz;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

constexpr int kMaxDevices = 64;

// Raises a kernel's dynamic shared-memory limit on the current device.  The
// attribute belongs to the device's context, so it is set once per device
// (bit `dev` of `done`); devices beyond 64 set it on every call.
template <typename Kern>
mla_status set_smem_limit(Kern kern, int smem, std::atomic<unsigned long long>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  const unsigned long long bit = dev >= 0 && dev < kMaxDevices ? 1ull << dev : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return MLA_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return MLA_ERR_CUDA;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return MLA_OK;
}

// Tile width, pipeline depth, K blocks per stage, CTA target and 128-row tiles
// per CTA (per-head modes) of one GEMM launch.
struct GemmConfig {
  int bn, stages, kbb, target_ctas, mt = 1;
};

template <int BN, bool AMN, int STAGES, int KBB, int MT = 1>
mla_status launch_tc(const GemmArgs& a, dim3 grid, cudaStream_t st, bool pdl) {
  using L = GemmSmem<BN, STAGES, KBB, MT>;
  constexpr int smem = L::kBytes;
  auto kern = gemm_tc_kernel<BN, AMN, STAGES, KBB, MT>;
  static std::atomic<unsigned long long> attr_done{0};
  const mla_status s = set_smem_limit(kern, smem, attr_done);
  if (s != MLA_OK) return s;
  if (a.cluster_k <= 1) return launch(kern, grid, dim3(192), smem, st, pdl, a);
  // the splits of a tile (grid z) form one cluster
  if (!L::kClusterK || a.cluster_k > kMaxClusterK || static_cast<int>(grid.z) != a.cluster_k)
    return MLA_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = a.cluster_k;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, a) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// The instantiated configurations (bn, stages, K blocks per stage).
template <bool AMN>
mla_status launch_tc_cfg(const GemmConfig& k, const GemmArgs& a, dim3 grid, cudaStream_t st, bool pdl) {
  if (k.mt == 4 && k.bn == 64 && k.stages == 2 && k.kbb == 1) return launch_tc<64, AMN, 2, 1, 4>(a, grid, st, pdl);
  if (k.mt == 2 && k.bn == 64 && k.stages == 2 && k.kbb == 1) return launch_tc<64, AMN, 2, 1, 2>(a, grid, st, pdl);
  if (k.mt != 1) return MLA_ERR_UNSUPPORTED;
#define MLA_GEMM_CFG(BN, S, KB) \
  if (k.bn == BN && k.stages == S && k.kbb == KB) return launch_tc<BN, AMN, S, KB>(a, grid, st, pdl);
  MLA_GEMM_CFG(32, 5, 1) MLA_GEMM_CFG(64, 4, 1) MLA_GEMM_CFG(128, 3, 1) MLA_GEMM_CFG(256, 4, 1)
  MLA_GEMM_CFG(32, 4, 2) MLA_GEMM_CFG(64, 4, 2) MLA_GEMM_CFG(32, 2, 4) MLA_GEMM_CFG(64, 2, 4)
  MLA_GEMM_CFG(64, 2, 2) MLA_GEMM_CFG(32, 2, 2) MLA_GEMM_CFG(128, 2, 2) MLA_GEMM_CFG(256, 2, 1)
#undef MLA_GEMM_CFG
  return MLA_ERR_UNSUPPORTED;
}

// Default configuration for N tokens: weight-streaming shapes (N <= 128)
// take 3-5 stages of one K block, larger N 256-wide tiles with two stages, so
// that two CTAs share an SM and one's epilogue (staged in column chunks)
// overlaps the other's MMAs.
GemmConfig choose_gemm_config(int N, int num_sms) {
  if (N <= 32) return {32, 5, 1, 2 * num_sms};
  if (N <= 64) return {64, 4, 1, 2 * num_sms};
  if (N <= 128) return {128, 3, 1, 2 * num_sms};
  return {256, 2, 1, 2 * num_sms};
}

mla_status run_gemm_tc(const Ctx& c, const GemmSpec& g, const GemmConfig& cfg) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  const int bn = cfg.bn;
  const int n_tiles = (g.N + bn - 1) / bn;
  a.mode = g.mode;
  a.N = g.N;
  a.boxB_rows = std::min(bn, g.N);
  a.kb_total = g.K / 64;
  a.head_rows = g.head_rows;
  a.b_head_stride = g.b_head_stride;
  a.status = c.status;
  a.tok = g.tok;
  a.x_independent = g.x_independent ? 1 : 0;
  int m_tiles = 0, mt_per_cta = 1;
  if (g.mode == GEMM_DENSE) {
    a.nseg = g.nseg;
    for (int s = 0; s < g.nseg; ++s) {
      a.seg_tile0[s] = m_tiles;
      m_tiles += (g.rows[s] + 127) / 128;
      a.seg_rows[s] = g.rows[s];
      a.boxA_rows[s] = std::min(128, g.rows[s]);
      a.epi[s] = g.epi[s];
      if (!make_map_2d(&a.mapA[s], g.A[s], g.K, g.rows[s], g.a_ld, a.boxA_rows[s])) return MLA_ERR_CUDA;
    }
    a.seg_tile0[g.nseg] = m_tiles;
  } else {
    const int tph = (g.rows[0] + 127) / 128;
    a.nseg = 1;
    a.seg_tile0[0] = 0;
    a.seg_tile0[1] = tph;
    a.seg_rows[0] = g.rows[0];
    a.epi[0] = g.epi[0];
    m_tiles = tph * g.heads;
    if (cfg.mt > 1 && tph % cfg.mt == 0) mt_per_cta = cfg.mt;
    if (g.mode == GEMM_HEAD_MNMAJOR) {
      a.boxA_rows[0] = 64;
      if (!make_map_2d(&a.mapA[0], g.A[0], g.a_ld, g.a_total_rows, g.a_ld, 64)) return MLA_ERR_CUDA;
    } else {
      a.boxA_rows[0] = 128;
      if (!make_map_2d(&a.mapA[0], g.A[0], g.K, g.a_total_rows, g.a_ld, 128)) return MLA_ERR_CUDA;
    }
  }
  if (!make_map_2d(&a.mapB, g.X, g.x_cols, g.N, g.x_ld, a.boxB_rows)) return MLA_ERR_CUDA;
  // split-K so that small tile counts still cover the SMs
  const int tiles = m_tiles * n_tiles;
  const int target = std::min(cfg.target_ctas, kMaxGemmCtas);
  int splits = 1;
  // per-head GEMMs (W_UV at n_h = 128) that already cover half the SMs run
  // without split-K: the partial round trip and second kernel cost more than
  // the extra parallelism gains
  const bool split_ok = g.mode == GEMM_DENSE || 2 * tiles <= c.num_sms;
  if (split_ok && mt_per_cta == 1 && n_tiles == 1 && tiles < target) {
    splits = std::max(1, std::min(a.kb_total / (2 * cfg.kbb), target / tiles));
  }
  int kbps = (a.kb_total + splits - 1) / splits;
  kbps = (kbps + cfg.kbb - 1) / cfg.kbb * cfg.kbb;  // whole stages per split
  splits = (a.kb_total + kbps - 1) / kbps;
  // Split-K inside clusters where the tile shape leaves room in shared memory
  // for the partial and staging tiles: the S splits of a tile (S a power of
  // two <= 8 that divides the K blocks into whole stages) sum their partials
  // through distributed shared memory, with no fp32 round trip through HBM and
  // no second kernel.
  const bool cluster_fits = mt_per_cta == 1 && cfg.stages * cfg.kbb * 16384 >= 2 * bn * 128 * 4;
  if (splits > 1 && cluster_fits) {
    int S = 1;
    while (2 * S <= kMaxClusterK && tiles * 2 * S <= target && a.kb_total % (2 * S * cfg.kbb) == 0) S *= 2;
    if (S > 1) {
      splits = S;
      kbps = a.kb_total / S;
      a.cluster_k = S;
    }
  }
  a.splits = splits;
  a.kb_per_split = kbps;
  a.partials = reinterpret_cast<float*>(c.ws + c.L.gpart);
  dim3 grid(m_tiles / mt_per_cta, n_tiles, splits);
  GemmConfig k = cfg;
  k.mt = mt_per_cta;
  mla_status s = g.mode == GEMM_HEAD_MNMAJOR ? launch_tc_cfg<true>(k, a, grid, c.st, c.pdl)
                                            : launch_tc_cfg<false>(k, a, grid, c.st, c.pdl);
  if (s != MLA_OK || splits == 1 || a.cluster_k > 1) return s;
  // split-K: a wide second kernel sums the partials in split order and runs the epilogue
  const dim3 rgrid(m_tiles, bn / 4);
  switch (bn) {
    case 32: return launch(gemm_splitk_epilogue_kernel<32>, rgrid, dim3(128), 0, c.st, c.pdl, a);
    case 64: return launch(gemm_splitk_epilogue_kernel<64>, rgrid, dim3(128), 0, c.st, c.pdl, a);
    case 128: return launch(gemm_splitk_epilogue_kernel<128>, rgrid, dim3(128), 0, c.st, c.pdl, a);
    default: return launch(gemm_splitk_epilogue_kernel<256>, rgrid, dim3(128), 0, c.st, c.pdl, a);
  }
}

template <typename T>
mla_status run_gemm_simt(const Ctx& c, const GemmSpec& g) {
  SimtGemmArgs a;
  memset(&a, 0, sizeof(a));
  int M = 0;
  if (g.mode == GEMM_DENSE) {
    a.nseg = g.nseg;
    for (int s = 0; s < g.nseg; ++s) {
      a.A[s] = g.A[s];
      a.seg_row0[s] = M;
      M += g.rows[s];
      a.epi[s] = g.epi[s];
    }
    a.seg_row0[g.nseg] = M;
    a.a_sm = g.a_ld;
    a.a_sk = 1;
    a.a_hoff = 0;
  } else {
    a.nseg = 1;
    a.A[0] = g.A[0];
    M = g.rows[0];
    a.seg_row0[0] = 0;
    a.seg_row0[1] = M;
    a.epi[0] = g.epi[0];
    a.a_hoff = static_cast<long long>(g.head_rows) * g.a_ld;
    if (g.mode == GEMM_HEAD_MNMAJOR) { a.a_sm = 1; a.a_sk = g.a_ld; }
    else { a.a_sm = g.a_ld; a.a_sk = 1; }
  }
  a.X = g.X;
  a.x_sn = g.x_ld;
  a.x_hoff = g.b_head_stride;
  a.M = M;
  a.N = g.N;
  a.K = g.K;
  a.heads = g.heads;
  a.tok = g.tok;
  a.status = c.status;
  dim3 grid((M + 31) / 32, (g.N + 7) / 8, g.heads);
  g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
  simt_gemm_kernel<T><<<grid, dim3(32, 8), 0, c.st>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

bool tc_gemm_ok(const mla_dims& d) {
  return d.dtype == MLA_BF16 && d.d_model % 64 == 0 && d.d_cq % 64 == 0 && d.d_c % 128 == 0 && d.d_h == 128 &&
         (d.n_h * d.d_h) % 64 == 0 && d.d_R % 8 == 0 && d.d_R <= 128;
}

mla_status run_gemm(const Ctx& c, const GemmSpec& g) {
  if (tc_gemm_ok(c.d)) {
    GemmConfig cfg = choose_gemm_config(g.N, c.num_sms);
    // per-head weight blocks of several 128-row tiles (W_UK^T: d_c rows per head)
    // share one X block: where the tiles fill the SMs twice over (V2's 128
    // heads), a CTA takes two of them, one accumulator each; fewer tiles
    // (V2-Lite's 16 heads) keep one per CTA, which measured 2 us faster there
    if (g.mode != GEMM_DENSE && g.N <= 64 && g.rows[0] % 512 == 0 && g.heads * (g.rows[0] / 128) >= 2 * c.num_sms)
      cfg = {64, 2, 1, c.num_sms, 2};
    return run_gemm_tc(c, g, cfg);
  }
  // fp32 storage (check_dims admits bf16 only with tensor-core shapes)
  return c.d.dtype == MLA_FP32 ? run_gemm_simt<float>(c, g) : MLA_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mla_status check_dims(const mla_dims* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->d_model <= 0 || d->n_h <= 0 || d->d_h <= 0 || d->d_R <= 0 || d->d_c <= 0 || d->d_cq < 0)
    return MLA_ERR_INVALID_ARG;
  if (!(d->rope_base > 1.0) || !std::isfinite(d->rope_base)) return MLA_ERR_INVALID_ARG;
  if (d->yarn_s != 0.0 &&
      (!(d->yarn_s >= 1.0) || !std::isfinite(d->yarn_s) || !(d->yarn_alpha >= 0.0) ||
       !(d->yarn_beta > d->yarn_alpha) || !std::isfinite(d->yarn_beta) || !(d->yarn_L0 > 0.0) ||
       !std::isfinite(d->yarn_L0)))
    return MLA_ERR_INVALID_ARG;
  if (d->dtype != MLA_BF16 && d->dtype != MLA_FP32) return MLA_ERR_UNSUPPORTED;
  if (d->cache_format != MLA_CACHE_DTYPE && d->cache_format != MLA_CACHE_E4M3) return MLA_ERR_UNSUPPORTED;
  if (d->cache_format == MLA_CACHE_E4M3 && d->dtype != MLA_BF16) return MLA_ERR_UNSUPPORTED;
  if (d->d_R % 2 != 0) return MLA_ERR_UNSUPPORTED;
  // CUDA-core kernels hold d_c/32 <= 16 latent columns and d_h/32 <= 8 value columns per lane.
  if (d->d_c > 512 || d->d_h > 256 || d->d_c % 4 != 0) return MLA_ERR_UNSUPPORTED;
  // 16-byte rows for every tensor the kernels load
  const int es = d->dtype == MLA_FP32 ? 4 : 2;
  if (row_bytes(*d) % 16 || (d->d_model * es) % 16 || (d->d_c * es) % 16) return MLA_ERR_UNSUPPORTED;
  // bf16 storage runs on the tensor-core kernels only, which are built for the
  // DeepSeek-V2 head shape (d_h = 128, d_R = 64, d_c = 512, up to 128 heads)
  // and 64-wide K blocks; the CUDA-core kernels serve fp32 storage alone.
  if (d->dtype == MLA_BF16 &&
      (d->d_h != 128 || d->d_R != 64 || d->d_c != 512 || d->n_h > 128 || d->d_model % 64 != 0 || d->d_cq % 64 != 0))
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

mla_status check_weights(const mla_dims* d, const mla_weights* w) {
  if (!w) return MLA_ERR_INVALID_ARG;
  const void* ps[] = {w->W_UQ, w->W_QR, w->W_DKV, w->W_UK, w->W_UV, w->W_KR, w->W_O};
  for (const void* p : ps) {
    if (!p) return MLA_ERR_INVALID_ARG;
    if (!aligned16(p)) return MLA_ERR_MISALIGNED;
  }
  if (d->d_cq) {
    if (!w->W_DQ) return MLA_ERR_INVALID_ARG;
    if (!aligned16(w->W_DQ)) return MLA_ERR_MISALIGNED;
  }
  if (w->g_q && !d->d_cq) return MLA_ERR_INVALID_ARG;  // no c^Q to normalise without query compression
  if ((w->g_kv && !aligned16(w->g_kv)) || (w->g_q && !aligned16(w->g_q))) return MLA_ERR_MISALIGNED;
  return MLA_OK;
}

mla_status check_cache(const mla_cache* c) {
  if (!c || !c->base || c->n_rows <= 0) return MLA_ERR_INVALID_ARG;
  if (c->block_table) {
    if (c->block_size <= 0 || c->block_size % 64 != 0 || c->max_blocks <= 0) return MLA_ERR_INVALID_ARG;
    if (!aligned16(c->block_table)) return MLA_ERR_MISALIGNED;
  } else if (!c->seq_start) {
    return MLA_ERR_INVALID_ARG;
  }
  if (!aligned16(c->base)) return MLA_ERR_MISALIGNED;
  return MLA_OK;
}

CacheLayout cache_layout(const mla_cache* c) {
  CacheLayout l{};
  l.seq_start = c->seq_start;
  l.block_table = c->block_table;
  l.block_size = c->block_table ? c->block_size : 0;
  l.max_blocks = c->block_table ? c->max_blocks : 0;
  return l;
}

enum Region { REGION_BASE, REGION_DECODE, REGION_PREFILL };

mla_status make_ctx(Ctx& c, const mla_dims* d, int max_batch, int max_tokens, Region region, void* ws,
                    size_t ws_bytes, mla_stream_t stream) {
  c.d = *d;
  c.L = make_layout(*d, max_batch, max_tokens);
  if (!ws) return MLA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return MLA_ERR_MISALIGNED;
  const size_t need = region == REGION_DECODE ? c.L.decode_end
                      : region == REGION_PREFILL ? c.L.prefill_end : c.L.base_end;
  if (ws_bytes < need) return MLA_ERR_WORKSPACE;
  c.ws = static_cast<uint8_t*>(ws);
  c.status = reinterpret_cast<int*>(c.ws + c.L.status);
  c.st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&c.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

TokenMap cache_tokens(const mla_dims& d, const mla_cache* cache) {
  TokenMap t{};
  t.lay = cache_layout(cache);
  t.capacity = cache->capacity;
  t.n_rows = cache->n_rows;
  t.cache = cache->base;
  t.row_bytes = row_bytes(d);
  t.kr_off = cache_fp8(d) ? d.d_c : d.d_c * elem_size(d);
  t.fp8 = cache_fp8(d) ? 1 : 0;
  t.d_c = d.d_c;
  t.d_R = d.d_R;
  t.log2_base = std::log2(d.rope_base);
  t.seq_const = -1;
  t.yarn_s = d.yarn_s;
  t.yarn_alpha = d.yarn_alpha;
  t.yarn_beta = d.yarn_beta;
  t.yarn_L0 = d.yarn_L0;
  return t;
}

// Fills the call's (cos, sin) table for T tokens and points `tk` at it.
mla_status launch_rope_table(const Ctx& c, TokenMap& tk, int T, void* table) {
  if (tk.d_R < 2 || T <= 0) return MLA_OK;
  const long long total = static_cast<long long>(T) * (tk.d_R / 2);
  const int blocks = static_cast<int>(std::min<long long>(4 * c.num_sms, (total + 255) / 256));
  const mla_status s = launch(rope_table_kernel, dim3(blocks), dim3(256), 0, c.st, c.pdl, tk, T,
                              reinterpret_cast<float2*>(table));
  if (s == MLA_OK) tk.rope = reinterpret_cast<const float2*>(table);
  return s;
}

Epi epi_store(void* out, long long ld, int col0, float scale, int out_f32 = 0) {
  Epi e{};
  e.kind = EPI_STORE;
  e.out = out;
  e.ld = ld;
  e.col0 = col0;
  e.scale = scale;
  e.out_f32 = out_f32;
  return e;
}
Epi epi_kind(int kind, void* out = nullptr, long long ld = 0, long long hs = 0, int col0 = 0, int dh = 0,
             float scale = 1.f) {
  Epi e{};
  e.kind = kind;
  e.out = out;
  e.ld = ld;
  e.hs = hs;
  e.col0 = col0;
  e.dh = dh;
  e.scale = scale;
  return e;
}

// Factor folded into the query: scores come out in log2 units (the softmax
// uses exp2) and carry the softmax scale 1/sqrt(d_h + d_R) ("DeepSeek-V2
// summary" App. C), times YaRN's t with sqrt(t) = 0.0707 ln s + 1 (§3.1.4).
float qlat_scale(const mla_dims& d) {
  double t = 1.0;
  if (d.yarn_s != 0.0) {
    const double rt = 0.0707 * std::log(d.yarn_s) + 1.0;
    t = rt * rt;
  }
  return static_cast<float>(1.4426950408889634 * t / std::sqrt(static_cast<double>(d.d_h + d.d_R)));
}

// Appends the [W_DKV; W_KR] segments (cache-row epilogues) to a dense GEMM.
// With an RMSNorm gain on c^KV, or an E4M3 cache, the W_DKV segment leaves
// c^KV in fp32 at `nkv` ([tokens x d_c]) for launch_latent_norm, which
// writes the cache rows' c^KV part.
void add_cache_segments(GemmSpec& g, const mla_dims& d, const mla_weights* w, void* nkv) {
  g.A[g.nseg] = w->W_DKV;
  g.rows[g.nseg] = d.d_c;
  g.epi[g.nseg] = (w->g_kv || cache_fp8(d)) ? epi_store(nkv, d.d_c, 0, 1.f, 1) : epi_kind(EPI_CACHE_CKV);
  ++g.nseg;
  g.A[g.nseg] = w->W_KR;
  g.rows[g.nseg] = d.d_R;
  g.epi[g.nseg] = epi_kind(EPI_CACHE_KR);
  ++g.nseg;
}

// RMSNorm of the latents of T tokens (no-op without gains): c^KV from `nkv`
// into the tokens' cache rows, c^Q from `nq` into `cq_out` (storage dtype).
mla_status launch_latent_norm(const Ctx& c, const mla_weights* w, const TokenMap& tk, int T, const void* nkv,
                              const void* nq, void* cq_out) {
  if (!w->g_kv && !w->g_q && !tk.fp8) return MLA_OK;
  const float* fk = (w->g_kv || tk.fp8) ? static_cast<const float*>(nkv) : nullptr;
  const float* fq = static_cast<const float*>(nq);
  if (c.d.dtype == MLA_FP32)
    return launch(latent_norm_kernel<float>, dim3(T), dim3(256), 0, c.st, c.pdl, fk,
                  static_cast<const float*>(w->g_kv), fq, static_cast<const float*>(w->g_q), c.d.d_cq,
                  static_cast<float*>(cq_out), tk, c.status);
  return launch(latent_norm_kernel<__nv_bfloat16>, dim3(T), dim3(256), 0, c.st, c.pdl, fk,
                static_cast<const __nv_bfloat16*>(w->g_kv), fq, static_cast<const __nv_bfloat16*>(w->g_q), c.d.d_cq,
                static_cast<__nv_bfloat16*>(cq_out), tk, c.status);
}

cudaEvent_t g_attn_begin = nullptr, g_attn_end = nullptr;  // diagnostic hook (mla_set_attention_events)

void attn_event(cudaEvent_t e, cudaStream_t st) {
  if (e) cudaEventRecord(e, st);
}

template <bool kFp8>
mla_status launch_attn_kernel(const AttnArgs& a, int W, cudaStream_t st, bool pdl) {
  static std::atomic<unsigned long long> attr_done{0};
  const mla_status s = set_smem_limit(attn_decode_tc_kernel<kFp8>, attn::Cfg<kFp8>::kSmem, attr_done);
  if (s != MLA_OK) return s;
  return launch(attn_decode_tc_kernel<kFp8>, dim3(2 * W), dim3(attn::Cfg<kFp8>::kThreads), attn::Cfg<kFp8>::kSmem, st,
                pdl, a);
}

bool attn_tc_ok(const mla_dims& d);

// Few heads (V2-Lite's 16) on bf16 rows take the single-CTA kernel with the
// tokens as the MMA's M dimension.
bool attn_sh_ok(const mla_dims& d) { return attn_tc_ok(d) && d.n_h <= attn_sh::kNH && !cache_fp8(d); }

mla_status launch_attn_decode_tc(const mla_dims& d, const __nv_bfloat16* qlat, const mla_cache* cache,
                                 const int32_t* seqlen, const int* tile_start, const int* seg_start, int B, int W,
                                 int n_h, float* o_part, float* ml, int* status, cudaStream_t st, bool pdl) {
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  if (cache->n_rows > (1ll << 31) - 128) return MLA_ERR_UNSUPPORTED;  // tile rows are int32 TMA coordinates
  const bool fp8 = cache_fp8(d);
  const int rb = row_bytes(d);
  // bf16 view of the rows (the whole row for bf16 rows; k^R for E4M3 rows)
  if (!make_map_2d(&a.map_cache, cache->base, rb / 2, cache->n_rows, rb / 2, attn::kHalf)) return MLA_ERR_CUDA;
  if (fp8) {
    if (!make_map_2d_u8(&a.map_code, cache->base, rb, cache->n_rows, rb, 256, attn::kHalf) ||
        !make_map_2d_u8(&a.map_scale, cache->base, rb, cache->n_rows, rb, 16, attn::kHalf))
      return MLA_ERR_CUDA;
    a.kr_x = d.d_c / 2;
    a.scale_x = d.d_c + 2 * d.d_R;
  }
  a.qlat = qlat;
  a.lay = cache_layout(cache);
  a.n_rows = cache->n_rows;
  a.seqlen = seqlen;
  a.tile_start = tile_start;
  a.seg_start = seg_start;
  a.B = B;
  a.W = W;
  a.n_h = n_h;
  a.o_part = o_part;
  a.ml_part = ml;
  a.status = status;
  if (fp8) return launch_attn_kernel<true>(a, W, st, pdl);
  if (attn_sh_ok(d)) {
    // few heads: one CTA per worker, tokens as the MMA's M
    static std::atomic<unsigned long long> attr_done{0};
    const mla_status s = set_smem_limit(attn_decode_sh_kernel, attn_sh::kSmem, attr_done);
    if (s != MLA_OK) return s;
    return launch(attn_decode_sh_kernel, dim3(W), dim3(attn_sh::kThreads), attn_sh::kSmem, st, pdl, a);
  }
  return launch_attn_kernel<false>(a, W, st, pdl);
}

bool prefill_tc_ok(const mla_dims& d) {
  return d.dtype == MLA_BF16 && d.d_h == 128 && d.d_R == 64 && tc_gemm_ok(d);
}

bool attn_tc_ok(const mla_dims& d) {
  return kAttnTcReady && d.dtype == MLA_BF16 && d.n_h <= 128 && d.d_c == 512 && d.d_R == 64;
}

// Attention workers of a decode call: one CTA per SM on the few-head kernel,
// one 2-CTA cluster per SM pair on the other tensor-core path, two CTAs per SM
// on the CUDA-core path.
int decode_workers(const mla_dims& d, int num_sms) {
  const int W = attn_sh_ok(d)   ? std::min(kMaxWorkers, num_sms)
                : attn_tc_ok(d) ? std::min(kMaxWorkers, num_sms / 2)
                                : std::min(kMaxWorkers, num_sms * 2);
  return W < 1 ? 1 : W;
}

// a6 + a7 in one kernel (tensor-core path): combine the attention partials
// into the W_UV product's B operand, o = W_UV_i o_lat_i, and write o_lat.
mla_status launch_uv_combine(const Ctx& c, const mla_weights* w, const float* opart, const float* ml,
                             const int* seg_start, int B, void* olat, void* o, const TokenMap& tk) {
  const mla_dims& d = c.d;
  const long long HD = static_cast<long long>(d.n_h) * d.d_h;
  UvCombineArgs a;
  memset(&a, 0, sizeof(a));
  if (!make_map_2d(&a.mapA, w->W_UV, d.d_c, HD, d.d_c, 128)) return MLA_ERR_CUDA;
  a.o_part = opart;
  a.ml_part = ml;
  a.seg_start = seg_start;
  a.n_h = d.n_h;
  a.N = B;
  // K splits: while the (head, 64-sequence) tiles would fill under half the
  // SMs, split each tile's 8 K blocks over a cluster of up to 4 (V2-Lite: 16 heads)
  const int tiles = d.n_h * ((B + 63) / 64);
  a.ks = 1;
  while (a.ks < uvc::kMaxKs && 2 * tiles * a.ks <= c.num_sms) a.ks *= 2;
  a.olat = static_cast<__nv_bfloat16*>(olat);
  a.epi = epi_kind(EPI_PER_HEAD, o, HD, d.d_h, 0, 0, 1.f);
  a.tok = tk;
  a.status = c.status;
  static std::atomic<unsigned long long> attr_done{0};
  const mla_status s = set_smem_limit(uv_combine_kernel, uvc::kSmem, attr_done);
  if (s != MLA_OK) return s;
  return launch_cluster_z(uv_combine_kernel, dim3(d.n_h, (B + 63) / 64, a.ks), dim3(uvc::kThreads), uvc::kSmem, c.st,
                          c.pdl, a.ks, a);
}

// The decode launch sequence (a1 .. a8 of the hot path) on an already checked
// context; shared by mla_decode and the no-allocation variant.
mla_status decode_run(Ctx& c, const mla_weights* w, const void* h, int B, const mla_cache* cache,
                      const int32_t* seqlen, float* u) {
  const mla_dims& d = c.d;
  mla_status s = MLA_OK;
  const int es = elem_size(d);
  const int row = row_elems(d);
  const long long HD = static_cast<long long>(d.n_h) * d.d_h;
  uint8_t* ws = c.ws;
  void* cq = ws + c.L.cq;
  void* qc = ws + c.L.qc;
  void* qlat = ws + c.L.qlat;
  void* olat = ws + c.L.olat;
  void* o = ws + c.L.o;
  int* tile_start = reinterpret_cast<int*>(ws + c.L.tile_start);
  int* seg_start = reinterpret_cast<int*>(ws + c.L.seg_start);
  const float qs = qlat_scale(d);
  TokenMap tk = cache_tokens(d, cache);
  tk.pos = seqlen;  // the new token of sequence b sits at position L_b
  (void)es;

  // ---- attention plan (device side: reads seqlen, no host sync) and the RoPE table of the new tokens
  const bool tc_attn = attn_tc_ok(d);
  const int tile_tokens = tc_attn ? kAttnTileTokens : 64;
  const int W = decode_workers(d, c.num_sms);
  c.pdl = tc_gemm_ok(d);
  float2* rope = d.d_R >= 2 ? reinterpret_cast<float2*>(ws + c.L.rope) : nullptr;
  if ((s = launch(plan_kernel, dim3(1), dim3(1024), 0, c.st, c.pdl, seqlen, B, tile_tokens, W, tile_start, seg_start,
                  c.status, tk, rope)) != MLA_OK)
    return s;
  tk.rope = rope;

  // ---- a1 (+a2): down-projections from h, cache append of the new token.
  // h is a call input, so the GEMM streams weights and h while the planner
  // runs and waits for it only in the epilogue (RoPE table, cache rows).
  {
    GemmSpec g;
    g.K = d.d_model;
    g.a_ld = d.d_model;
    g.X = h;
    g.x_independent = true;
    g.x_cols = d.d_model;
    g.x_ld = d.d_model;
    g.N = B;
    g.tok = tk;
    if (d.d_cq) {
      g.A[0] = w->W_DQ;
      g.rows[0] = d.d_cq;
      g.epi[0] = w->g_q ? epi_store(ws + c.L.nq, d.d_cq, 0, 1.f, 1) : epi_store(cq, d.d_cq, 0, 1.f);
      g.nseg = 1;
    } else {
      g.A[0] = w->W_UQ;
      g.rows[0] = static_cast<int>(HD);
      g.epi[0] = epi_store(qc, HD, 0, 1.f);
      g.A[1] = w->W_QR;
      g.rows[1] = d.n_h * d.d_R;
      g.epi[1] = epi_kind(EPI_QLAT_ROPE, qlat, static_cast<long long>(d.n_h) * row, row, 0, 0, qs);
      g.nseg = 2;
    }
    add_cache_segments(g, d, w, ws + c.L.nkv);
    if ((s = run_gemm(c, g)) != MLA_OK) return s;
    if ((s = launch_latent_norm(c, w, tk, B, ws + c.L.nkv, ws + c.L.nq, cq)) != MLA_OK) return s;
  }
  // ---- a3: query up-projection from c^Q (+ RoPE on q^R)
  if (d.d_cq) {
    GemmSpec g;
    g.K = d.d_cq;
    g.a_ld = d.d_cq;
    g.X = cq;
    g.x_cols = d.d_cq;
    g.x_ld = d.d_cq;
    g.N = B;
    g.tok = tk;
    g.A[0] = w->W_UQ;
    g.rows[0] = static_cast<int>(HD);
    g.epi[0] = epi_store(qc, HD, 0, 1.f);
    g.A[1] = w->W_QR;
    g.rows[1] = d.n_h * d.d_R;
    g.epi[1] = epi_kind(EPI_QLAT_ROPE, qlat, static_cast<long long>(d.n_h) * row, row, 0, 0, qs);
    g.nseg = 2;
    if ((s = run_gemm(c, g)) != MLA_OK) return s;
  }
  // ---- a4: absorb W_UK into the query: q_abs_i = W_UK_i^T q^C_i
  {
    GemmSpec g;
    g.mode = GEMM_HEAD_MNMAJOR;
    g.A[0] = w->W_UK;
    g.rows[0] = d.d_c;
    g.a_ld = d.d_c;
    g.a_total_rows = HD;
    g.K = d.d_h;
    g.X = qc;
    g.x_cols = HD;
    g.x_ld = HD;
    g.N = B;
    g.heads = d.n_h;
    g.head_rows = d.d_h;
    g.b_head_stride = d.d_h;
    g.tok = tk;
    g.epi[0] = epi_kind(EPI_PER_HEAD, qlat, static_cast<long long>(d.n_h) * row, row, 0, 0, qs);
    g.nseg = 1;
    if ((s = run_gemm(c, g)) != MLA_OK) return s;
  }
  // ---- a5: attention over the latent cache -> per-piece partials;  a6: combine
  float* opart = reinterpret_cast<float*>(ws + c.L.opart);
  float* ml = reinterpret_cast<float*>(ws + c.L.ml);
  attn_event(g_attn_begin, c.st);
  if (tc_attn) {
    if ((s = launch_attn_decode_tc(d, reinterpret_cast<const __nv_bfloat16*>(qlat), cache, seqlen, tile_start,
                                   seg_start, B, W, d.n_h, opart, ml, c.status, c.st, c.pdl)) != MLA_OK)
      return s;
  } else {
    if (d.dtype != MLA_FP32) return MLA_ERR_UNSUPPORTED;  // bf16 is on the tensor-core kernel alone
    const size_t shm = (row + 4 * d.d_c + 8) * sizeof(float);
    dim3 grid(W, d.n_h);
    g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
    simt_decode_attn_kernel<float><<<grid, 128, shm, c.st>>>(
        static_cast<const float*>(qlat), static_cast<const float*>(cache->base), cache_layout(cache), seqlen,
        tile_start, seg_start, B, W, d.n_h, d.d_c, d.d_R, tile_tokens, opart, ml);
    if (cudaPeekAtLastError() != cudaSuccess) return MLA_ERR_CUDA;
  }
  attn_event(g_attn_end, c.st);
  if (tc_attn && tc_gemm_ok(d)) {
    // ---- a6 + a7 fused: the combine feeds the absorbed W_UV product directly
    if ((s = launch_uv_combine(c, w, opart, ml, seg_start, B, olat, o, tk)) != MLA_OK) return s;
  } else {
    // fp32 storage (bf16 is on the tensor-core kernels alone): a separate combine, then W_UV
    if (d.dtype != MLA_FP32) return MLA_ERR_UNSUPPORTED;
    dim3 grid(B, (d.n_h + 3) / 4);  // one warp per (sequence, head)
    if ((s = launch(combine_kernel<float>, grid, dim3(128), 0, c.st, c.pdl, opart, ml, seg_start, d.n_h, d.d_c,
                    static_cast<float*>(olat))) != MLA_OK)
      return s;
    // ---- a7: absorbed W_UV on the latent output: o_i = W_UV_i o_lat_i
    GemmSpec g;
    g.mode = GEMM_HEAD_KMAJOR;
    g.A[0] = w->W_UV;
    g.rows[0] = d.d_h;
    g.a_ld = d.d_c;
    g.a_total_rows = HD;
    g.K = d.d_c;
    g.X = olat;
    g.x_cols = static_cast<long long>(d.n_h) * d.d_c;
    g.x_ld = g.x_cols;
    g.N = B;
    g.heads = d.n_h;
    g.head_rows = d.d_h;
    g.b_head_stride = d.d_c;
    g.tok = tk;
    g.epi[0] = epi_kind(EPI_PER_HEAD, o, HD, d.d_h, 0, 0, 1.f);
    g.nseg = 1;
    if ((s = run_gemm(c, g)) != MLA_OK) return s;
  }
  // ---- a8: u = W_O o
  {
    GemmSpec g;
    g.A[0] = w->W_O;
    g.rows[0] = d.d_model;
    g.a_ld = HD;
    g.K = static_cast<int>(HD);
    g.X = o;
    g.x_cols = HD;
    g.x_ld = HD;
    g.N = B;
    g.tok = tk;
    g.epi[0] = epi_store(u, d.d_model, 0, 1.f, 1);
    g.nseg = 1;
    if ((s = run_gemm(c, g)) != MLA_OK) return s;
  }
  return MLA_OK;
}

// One CTA whose thread 0 waits on a barrier nothing will complete: the
// bounded wait gives up after its time limit and records FAULT_WAIT_TIMEOUT.
// No load, store or MMA is in flight, so nothing lands after the CTA exits.
__global__ void wait_timeout_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx wc{status, &abort_flag};
    mbar_wait(&bar, 0, wc);
  }
  __syncthreads();
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

mla_status mla_check_wait_timeout(void* workspace, mla_stream_t stream) {
  if (!workspace) return MLA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return MLA_ERR_MISALIGNED;
  g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
  wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<int*>(workspace));
  return cudaPeekAtLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

unsigned long long mla_kernel_launches(void) { return g_kernel_launches.load(std::memory_order_relaxed); }

void mla_set_attention_events(void* begin, void* end) {
  g_attn_begin = static_cast<cudaEvent_t>(begin);
  g_attn_end = static_cast<cudaEvent_t>(end);
}

size_t mla_workspace_bytes(const mla_dims* dims, int max_batch, int max_tokens) {
  if (check_dims(dims) != MLA_OK) return 0;
  const Layout L = make_layout(*dims, max_batch, max_tokens);
  return std::max(L.decode_end, L.prefill_end);
}

size_t mla_workspace_offset(const mla_dims* dims, int max_batch, int max_tokens, int which) {
  if (check_dims(dims) != MLA_OK) return static_cast<size_t>(-1);
  const Layout L = make_layout(*dims, max_batch, max_tokens);
  switch (which) {
    case 0: return L.cq;
    case 1: return L.qc;
    case 2: return L.qlat;
    case 3: return L.olat;
    case 4: return L.o;
    case 5: return L.p_nkv;
    default: return static_cast<size_t>(-1);
  }
}

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported dims or dtype";
    case MLA_ERR_MISALIGNED: return "pointer not 16-byte aligned (workspace: 256-byte)";
    case MLA_ERR_WORKSPACE: return "workspace missing or too small";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_DEVICE_FAULT: return "device fault reported by a kernel";
  }
  return "unknown status";
}

mla_status mla_get_device_status(void* workspace, mla_stream_t stream, int* detail) {
  if (!workspace) return MLA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  // the status word is the first int of every layout
  if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MLA_ERR_CUDA;
  if (detail) *detail = v;
  if (v != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(int), st) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MLA_ERR_CUDA;
    return MLA_ERR_DEVICE_FAULT;
  }
  return MLA_OK;
}

mla_status mla_cache_append(const mla_dims* dims, const mla_weights* w, const void* h, int T, const int32_t* seq_idx,
                            const int32_t* pos, const mla_cache* cache, void* workspace, size_t workspace_bytes,
                            mla_stream_t stream) {
  mla_status s = check_dims(dims);
  if (s != MLA_OK) return s;
  if ((s = check_weights(dims, w)) != MLA_OK) return s;
  if ((s = check_cache(cache)) != MLA_OK) return s;
  if (T < 0) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!h || !seq_idx || !pos) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h)) return MLA_ERR_MISALIGNED;
  Ctx c;
  // with an RMSNorm on c^KV or an E4M3 cache the raw latents of the T tokens
  // need the prefill region
  const bool raw_ckv = w->g_kv || cache_fp8(*dims);
  if ((s = make_ctx(c, dims, 1, T, raw_ckv ? REGION_PREFILL : REGION_BASE, workspace, workspace_bytes, stream)) !=
      MLA_OK)
    return s;
  const mla_dims& d = *dims;
  GemmSpec g;
  g.K = d.d_model;
  g.a_ld = d.d_model;
  g.X = h;
  g.x_cols = d.d_model;
  g.x_ld = d.d_model;
  g.N = T;
  g.tok = cache_tokens(d, cache);
  g.tok.pos = pos;
  g.tok.seq = seq_idx;
  add_cache_segments(g, d, w, c.ws + c.L.p_nkv);
  if ((s = run_gemm(c, g)) != MLA_OK) return s;
  if (!raw_ckv) return MLA_OK;
  mla_weights kv_only = *w;
  kv_only.g_q = nullptr;  // appending caches c^KV only
  return launch_latent_norm(c, &kv_only, g.tok, T, c.ws + c.L.p_nkv, nullptr, nullptr);
}

mla_status mla_decode(const mla_dims* dims, const mla_weights* w, const void* h, int B, const mla_cache* cache,
                      const int32_t* seqlen, float* u, void* workspace, size_t workspace_bytes, mla_stream_t stream) {
  mla_status s = check_dims(dims);
  if (s != MLA_OK) return s;
  if ((s = check_weights(dims, w)) != MLA_OK) return s;
  if ((s = check_cache(cache)) != MLA_OK) return s;
  if (B <= 0 || !h || !seqlen || !u) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(u)) return MLA_ERR_MISALIGNED;
  Ctx c;
  if ((s = make_ctx(c, dims, B, 1, REGION_DECODE, workspace, workspace_bytes, stream)) != MLA_OK) return s;
  return decode_run(c, w, h, B, cache, seqlen, u);
}

}  // extern "C"

namespace {

// Copies the first nrows cache rows of sequence `seq` (contiguous or paged)
// into one contiguous block, 16 bytes per thread and step (row_bytes is a
// multiple of 16).
__global__ void gather_rows_kernel(const uint8_t* __restrict__ cache, const CacheLayout lay, int seq, long long nrows,
                                   int row_bytes, uint8_t* __restrict__ out) {
  const int v = row_bytes >> 4;  // 16-byte pieces per row
  const long long n = nrows * v;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / v;
    const int q = static_cast<int>(i - r * v);
    const long long src = lay.row(seq, r);  // negative: no page (reported by the call's cache write)
    reinterpret_cast<uint4*>(out)[i] =
        src < 0 ? make_uint4(0, 0, 0, 0)
                : *reinterpret_cast<const uint4*>(cache + src * row_bytes + static_cast<long long>(q) * 16);
  }
}

}  // namespace

extern "C" mla_status mla_prefill(const mla_dims* dims, const mla_weights* w, const void* h, int T, int start_pos,
                                  const mla_cache* cache, int seq, float* u, void* workspace, size_t workspace_bytes,
                                  mla_stream_t stream) {
  mla_status s = check_dims(dims);
  if (s != MLA_OK) return s;
  if ((s = check_weights(dims, w)) != MLA_OK) return s;
  if ((s = check_cache(cache)) != MLA_OK) return s;
  if (T <= 0 || start_pos < 0 || seq < 0 || !h || !u) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(u)) return MLA_ERR_MISALIGNED;
  if (cache_fp8(*dims)) return MLA_ERR_UNSUPPORTED;  // prefill reads and writes storage-dtype rows only
  const int S = start_pos + T;  // keys of the last token
  Ctx c;
  if ((s = make_ctx(c, dims, 1, S, REGION_PREFILL, workspace, workspace_bytes, stream)) != MLA_OK) return s;
  const mla_dims& d = *dims;
  const int row = row_elems(d);
  const int dq = d.d_h + d.d_R;
  const long long HD = static_cast<long long>(d.n_h) * d.d_h;
  uint8_t* ws = c.ws;
  void* cq = ws + c.L.p_cq;
  void* qp = ws + c.L.p_qp;
  void* rows = ws + c.L.p_rows;
  void* kc = ws + c.L.p_kc;
  void* vv = ws + c.L.p_v;
  void* att = ws + c.L.p_out;
  const float qs = qlat_scale(d);
  TokenMap tk = cache_tokens(d, cache);
  tk.pos_base = start_pos;
  tk.seq_const = seq;
  if ((s = launch_rope_table(c, tk, T, ws + c.L.p_rope)) != MLA_OK) return s;
  // ---- p1: down-projections and cache rows of the T new tokens
  {
    GemmSpec g;
    g.K = d.d_model;
    g.a_ld = d.d_model;
    g.X = h;
    g.x_cols = d.d_model;
    g.x_ld = d.d_model;
    g.N = T;
    g.tok = tk;
    if (d.d_cq) {
      g.A[0] = w->W_DQ;
      g.rows[0] = d.d_cq;
      g.epi[0] = w->g_q ? epi_store(ws + c.L.p_nq, d.d_cq, 0, 1.f, 1) : epi_store(cq, d.d_cq, 0, 1.f);
      g.nseg = 1;
    } else {
      g.A[0] = w->W_UQ;
      g.rows[0] = static_cast<int>(HD);
      g.epi[0] = epi_kind(EPI_HEADS, qp, static_cast<long long>(d.n_h) * dq, dq, 0, d.d_h, qs);
      g.A[1] = w->W_QR;
      g.rows[1] = d.n_h * d.d_R;
      g.epi[1] = epi_kind(EPI_QP_ROPE, qp, static_cast<long long>(d.n_h) * dq, dq, d.d_h, 0, qs);
      g.nseg = 2;
    }
    add_cache_segments(g, d, w, ws + c.L.p_nkv);
    if ((s = run_gemm(c, g)) != MLA_OK) return s;
    if ((s = launch_latent_norm(c, w, tk, T, ws + c.L.p_nkv, ws + c.L.p_nq, cq)) != MLA_OK) return s;
  }
  // ---- p2: queries [q^C ; RoPE(q^R)] per head
  if (d.d_cq) {
    GemmSpec g;
    g.K = d.d_cq;
    g.a_ld = d.d_cq;
    g.X = cq;
    g.x_cols = d.d_cq;
    g.x_ld = d.d_cq;
    g.N = T;
    g.tok = tk;
    g.A[0] = w->W_UQ;
    g.rows[0] = static_cast<int>(HD);
    g.epi[0] = epi_kind(EPI_HEADS, qp, static_cast<long long>(d.n_h) * dq, dq, 0, d.d_h, qs);
    g.A[1] = w->W_QR;
    g.rows[1] = d.n_h * d.d_R;
    g.epi[1] = epi_kind(EPI_QP_ROPE, qp, static_cast<long long>(d.n_h) * dq, dq, d.d_h, 0, qs);
    g.nseg = 2;
    if ((s = run_gemm(c, g)) != MLA_OK) return s;
  }
  // ---- the sequence's cache rows (prefix + new) as one contiguous block
  {
    const int row_bytes = row * elem_size(d);
    const int blocks = static_cast<int>(std::min<long long>(8 * c.num_sms, (static_cast<long long>(S) * (row_bytes / 16) + 255) / 256));
    g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
    gather_rows_kernel<<<blocks, 256, 0, c.st>>>(static_cast<const uint8_t*>(cache->base), cache_layout(cache), seq, S,
                                                 row_bytes, static_cast<uint8_t*>(rows));
    if (cudaPeekAtLastError() != cudaSuccess) return MLA_ERR_CUDA;
  }
  // ---- p3: un-absorbed keys and values of every key token: K^C = W_UK c, V = W_UV c
  {
    GemmSpec g;
    g.K = d.d_c;
    g.a_ld = d.d_c;
    g.X = rows;
    g.x_cols = row;
    g.x_ld = row;
    g.N = S;
    g.tok = tk;
    g.A[0] = w->W_UK;
    g.rows[0] = static_cast<int>(HD);
    g.epi[0] = epi_store(kc, HD, 0, 1.f);
    g.A[1] = w->W_UV;
    g.rows[1] = static_cast<int>(HD);
    g.epi[1] = epi_store(vv, HD, 0, 1.f);
    g.nseg = 2;
    if ((s = run_gemm(c, g)) != MLA_OK) return s;
  }
  // ---- p4: causal attention per head
  attn_event(g_attn_begin, c.st);
  if (prefill_tc_ok(d)) {
    PrefillArgs a;
    memset(&a, 0, sizeof(a));
    if (!make_map_2d(&a.map_q, qp, static_cast<long long>(d.n_h) * dq, T, static_cast<long long>(d.n_h) * dq, 128) ||
        !make_map_2d(&a.map_kc, kc, HD, S, HD, 128) || !make_map_2d(&a.map_kr, rows, row, S, row, 128) ||
        !make_map_2d(&a.map_v, vv, HD, S, HD, 128))
      return MLA_ERR_CUDA;
    a.out = static_cast<__nv_bfloat16*>(att);
    a.T = T;
    a.start_pos = start_pos;
    a.n_h = d.n_h;
    a.n_qt = (T + pf::kQ - 1) / pf::kQ;
    a.status = c.status;
    static std::atomic<unsigned long long> attr_done{0};
    if ((s = set_smem_limit(attn_prefill_tc_kernel, pf::kSmem, attr_done)) != MLA_OK) return s;
    g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
    attn_prefill_tc_kernel<<<dim3(a.n_qt, d.n_h), pf::kThreads, pf::kSmem, c.st>>>(a);
    if (cudaPeekAtLastError() != cudaSuccess) return MLA_ERR_CUDA;
  } else {
    if (d.dtype != MLA_FP32) return MLA_ERR_UNSUPPORTED;  // bf16 is on the tensor-core kernel alone
    const size_t shm = (dq + 4 * d.d_h + 8) * sizeof(float);
    dim3 grid(T, d.n_h);
    g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
    simt_prefill_attn_kernel<float><<<grid, 128, shm, c.st>>>(
        static_cast<const float*>(qp), static_cast<const float*>(kc), static_cast<const float*>(vv),
        static_cast<const float*>(rows), T, start_pos, d.n_h, d.d_h, d.d_R, d.d_c, static_cast<float*>(att));
    if (cudaPeekAtLastError() != cudaSuccess) return MLA_ERR_CUDA;
  }
  attn_event(g_attn_end, c.st);
  // ---- p5: u = W_O o
  {
    GemmSpec g;
    g.A[0] = w->W_O;
    g.rows[0] = d.d_model;
    g.a_ld = HD;
    g.K = static_cast<int>(HD);
    g.X = att;
    g.x_cols = HD;
    g.x_ld = HD;
    g.N = T;
    g.tok = tk;
    g.epi[0] = epi_store(u, d.d_model, 0, 1.f, 1);
    g.nseg = 1;
    if ((s = run_gemm(c, g)) != MLA_OK) return s;
  }
  return MLA_OK;
}

// ====================================================================== decode without a workspace
// Scratch of mla_decode_static: one file-scope device array per GPU that loads
// this library, held until the process exits.  Host code must not pass the
// array's name to a kernel (on the host it is only a stand-in); the device
// address comes from cudaGetSymbolAddress, looked up once per device.
namespace {

static __device__ __align__(256) uint8_t g_static_scratch[MLA_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

mla_status static_scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" mla_status mla_decode_static(const mla_dims* dims, const mla_weights* w, const void* h, int B,
                                        const mla_cache* cache, const int32_t* seqlen, float* u,
                                        mla_stream_t stream) {
  mla_status s = check_dims(dims);
  if (s != MLA_OK) return s;
  if ((s = check_weights(dims, w)) != MLA_OK) return s;
  if ((s = check_cache(cache)) != MLA_OK) return s;
  if (B <= 0 || !h || !seqlen || !u) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(u)) return MLA_ERR_MISALIGNED;
  Ctx c;
  c.d = *dims;
  c.st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&c.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MLA_ERR_CUDA;
  // exactly the space this batch uses on this device: split-K tiles of the
  // batch's width, attention partials for B + (workers on this GPU) slots
  c.L = make_layout_sized(*dims, B, 1, pick_bn(B), decode_workers(*dims, c.num_sms));
  if (c.L.decode_end > MLA_STATIC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((s = static_scratch_address(dev, &scratch)) != MLA_OK) return s;
  c.ws = static_cast<uint8_t*>(scratch);
  c.status = reinterpret_cast<int*>(c.ws + c.L.status);
  // the array keeps the previous call's contents: only the status word has to
  // start at zero (cleared here); every other region is written in full by a
  // kernel of this call before any kernel reads it
  if (cudaMemsetAsync(c.status, 0, sizeof(int), c.st) != cudaSuccess) return MLA_ERR_CUDA;
  return decode_run(c, w, h, B, cache, seqlen, u);
}
