// gemm_tc.cuh -- tcgen05 tensor-core GEMM used for every projection of the
// MLA path (W_DQ/W_DKV/W_KR, W_UQ/W_QR, the absorbed W_UK and W_UV, W_O, and
// the prefill key/value up-projection).
//
//   y[m, n] = sum_k A[m, k] * X[n, k]      A: weight rows (out features), X: tokens
//
// "Swap-AB" orientation: the weight is the M=128 operand and the tokens are
// the N operand (N = 32..256), so decode batches of 32-128 tokens still use
// full-rate M=128 MMAs and the kernel streams the weights at HBM speed.
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues tcgen05.mma, warps 2-5 run the epilogue (one TMEM lane per thread),
// staged in the idle pipeline buffers (in column chunks when the whole tile
// does not fit).
// Split-K: where the tile shape leaves room, the splits of a tile run as one
// cluster and sum their fp32 partials through distributed shared memory;
// otherwise they write fp32 partials and a second, wide kernel
// (gemm_splitk_epilogue_kernel) sums them.  Either way the sum runs in split
// order, so results do not depend on scheduling.
#pragma once
#include "epilogue.cuh"

namespace mla {

enum GemmMode : int {
  GEMM_DENSE = 0,        // A = one of up to 4 weight segments, K-major
  GEMM_HEAD_KMAJOR = 1,  // per-head A block rows [head*head_rows, +head_rows), K-major (W_UV)
  GEMM_HEAD_MNMAJOR = 2, // per-head A = W[head*head_rows + k, m]: M contiguous (W_UK^T)
};

constexpr int kMaxSeg = 4;
constexpr int kMaxClusterK = 8;  // splits of one tile reduced inside a cluster (portable cluster size)

struct GemmArgs {
  CUtensorMap mapA[kMaxSeg];
  CUtensorMap mapB;
  int mode;
  int nseg;
  int seg_tile0[kMaxSeg + 1];  // first M tile of each segment (cumulative); per-head modes: [0, tiles/head]
  int seg_rows[kMaxSeg];       // valid rows of each segment (per-head modes: rows of one head's output)
  int boxA_rows[kMaxSeg];      // TMA box rows of each A segment (K-major: min(128, rows))
  Epi epi[kMaxSeg];
  int head_rows;               // per-head modes: A rows per head along the K (MN-major) or M (K-major) axis
  int b_head_stride;           // per-head modes: column offset of a head's K range inside X
  int N;                       // tokens
  int boxB_rows;               // TMA box rows of X (min(BN, N))
  int kb_total;                // K / 64
  int kb_per_split;
  int splits;
  int cluster_k;               // > 1: the splits of a tile form one cluster and reduce through shared memory
  float* partials;             // [tiles][splits][BN/4][128][4] fp32 (splits > 1, cluster_k <= 1)
  int* status;
  int x_independent;           // 1: X is a call input no earlier kernel writes; only the epilogue waits
  TokenMap tok;
};

// One pipeline stage holds KBB consecutive 64-wide K blocks of A (MT tiles of
// 128 rows) and of X (BN rows): fewer, larger stages mean fewer barrier round
// trips and longer runs of each weight row in flight.
template <int BN, int STAGES, int KBB, int MT = 1>
struct GemmSmem {
  static constexpr int kSlabA = 16384;     // 128 rows x 128 B
  static constexpr int kSlabB = BN * 128;  // BN rows x 128 B
  static constexpr int kA = KBB * MT * kSlabA;
  static constexpr int kB = KBB * kSlabB;
  static constexpr int kStage = kA + kB;
  static constexpr int kBytes = 1024 + STAGES * kStage + 256;
  // cluster split-K keeps the fp32 partial tile and a staging tile in the A buffers
  static constexpr bool kClusterK = MT == 1 && STAGES * kA >= 2 * BN * 128 * 4;
  // token columns the idle pipeline buffers stage at once (fp32 staging): all
  // BN, or the largest power of two that fits
  static constexpr int stage_cols() {
    int c = BN;
    while (c > 16 && c * 128 * 4 > STAGES * kStage) c /= 2;
    return c;
  }
  static constexpr int kStageCols = stage_cols();
};

// MT > 1 (per-head modes, no split-K): one CTA computes MT consecutive
// 128-row tiles of a head against the same X block, one TMEM accumulator each.
template <int BN, bool A_MN, int STAGES, int KBB, int MT = 1>
__global__ void __launch_bounds__(192, 1) gemm_tc_kernel(const __grid_constant__ GemmArgs args) {
  using L = GemmSmem<BN, STAGES, KBB, MT>;
  static_assert(L::kStageCols * 128 * 4 <= STAGES * L::kStage && BN % L::kStageCols == 0,
                "the pipeline stages hold the fp32 staging tile, whole or in column chunks");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::kA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * L::kB);
  uint64_t* empty = full + STAGES;
  uint64_t* accum = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr uint32_t kTmemCols = BN * MT < 32 ? 32 : BN * MT;
  static_assert(BN * MT <= 512 && (BN * MT & (BN * MT - 1)) == 0, "TMEM columns: a power of two <= 512");

  // ---- which tile.  With several token tiles (prefill, long appends) the
  // grid is walked in groups of kRasterGroup weight tiles: consecutive CTAs
  // take the same few weight tiles against successive token tiles, so a
  // weight tile is read from HBM once and then from L2, instead of once per
  // token tile when all weight tiles run before the next token tile.
  int mt = blockIdx.x, nt = blockIdx.y;
  const int split = blockIdx.z;
  if (gridDim.y > 1) {
    constexpr int kRasterGroup = 8;
    const int num_m = gridDim.x, num_n = gridDim.y;
    const int lin = blockIdx.x + num_m * blockIdx.y;
    const int group = lin / (kRasterGroup * num_n);
    const int first_m = group * kRasterGroup;
    const int gm = min(num_m - first_m, kRasterGroup);  // weight tiles in this group
    const int in_group = lin - group * kRasterGroup * num_n;
    mt = first_m + in_group % gm;
    nt = in_group / gm;
  }
  int seg = 0, head = 0, m0;
  if (args.mode == GEMM_DENSE) {
    while (seg + 1 < args.nseg && mt >= args.seg_tile0[seg + 1]) ++seg;
    m0 = (mt - args.seg_tile0[seg]) * 128;
  } else {
    const int tph = args.seg_tile0[1];
    head = (mt * MT) / tph;
    m0 = ((mt * MT) % tph) * 128;
  }
  const int kb0 = split * args.kb_per_split;
  const int kb1 = min(args.kb_total, kb0 + args.kb_per_split);
  const int nkb = kb1 - kb0;                 // K blocks of this CTA
  const int nk = (nkb + KBB - 1) / KBB;      // pipeline stages of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&args.mapA[seg]);
    prefetch_tmap(&args.mapB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wc{args.status, abort_flag};

  if (threadIdx.x == 0) griddep_launch_dependents();
  if (warp == 0) {
    if (elect_one()) {
      const uint64_t polA = policy_evict_first();
      const uint64_t polB = policy_evict_last();
      const uint32_t bytesA = MT * (A_MN ? 16384u : static_cast<uint32_t>(args.boxA_rows[seg]) * 128u);
      const uint32_t bytesB = static_cast<uint32_t>(args.boxB_rows) * 128u;
      auto stage_kbs = [&](int i) { return min(KBB, nkb - i * KBB); };
      auto load_a = [&](int i, int j) {
        const int s = i % STAGES;
        const int kb = kb0 + i * KBB + j;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          uint8_t* a = sA + s * L::kA + (j * MT + t) * L::kSlabA;
          const int mr = m0 + t * 128;
          if (A_MN) {
            const int y = head * args.head_rows + kb * 64;
            tma_load_2d(a, &args.mapA[0], &full[s], mr, y, polA);
            tma_load_2d(a + 8192, &args.mapA[0], &full[s], mr + 64, y, polA);
          } else if (args.mode == GEMM_HEAD_KMAJOR) {
            tma_load_2d(a, &args.mapA[0], &full[s], kb * 64, head * args.head_rows + mr, polA);
          } else {
            tma_load_2d(a, &args.mapA[seg], &full[s], kb * 64, mr, polA);
          }
        }
      };
      auto load_b = [&](int i, int j) {
        const int s = i % STAGES;
        tma_load_2d(sB + s * L::kB + j * L::kSlabB, &args.mapB, &full[s],
                    head * args.b_head_stride + (kb0 + i * KBB + j) * 64, nt * BN, polB);
      };
      // Weights do not depend on earlier kernels: the first stages of A are
      // fetched before waiting for the kernel that produces X (no wait at all
      // when X is a call input).
      const int pre = nk < STAGES ? nk : STAGES;
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], stage_kbs(i) * (bytesA + bytesB));
        for (int j = 0; j < stage_kbs(i); ++j) load_a(i, j);
      }
      if (!args.x_independent) griddep_wait();
      for (int i = 0; i < pre; ++i)
        for (int j = 0; j < stage_kbs(i); ++j) load_b(i, j);
      int issued = pre;
      for (int i = pre; i < nk; ++i, ++issued) {
        const int s = i % STAGES;
        if (!mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, wc)) break;
        mbar_arrive_expect_tx(&full[s], stage_kbs(i) * (bytesA + bytesB));
        for (int j = 0; j < stage_kbs(i); ++j) {
          load_a(i, j);
          load_b(i, j);
        }
      }
      drain_ring(full, STAGES, issued);  // every issued load has landed before the CTA may leave
    }
  } else if (warp == 1) {
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_bf16(128, BN, A_MN, false);
      for (int i = 0; i < nk; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&full[s], ph, wc)) break;
        tc_fence_after();
        const int kbs = min(KBB, nkb - i * KBB);
        for (int j = 0; j < kbs; ++j) {
          const uint32_t b_base = smem_u32(sB + s * L::kB + j * L::kSlabB);
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const uint32_t a_base = smem_u32(sA + s * L::kA + (j * MT + t) * L::kSlabA);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t ad = A_MN ? sdesc_sw128(a_base + k * 2048, 8192, 1024) : sdesc_sw128(a_base + k * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(b_base + k * 32, 16, 1024);
              mma_ss(tmem + t * BN, ad, bd, idesc, (i > 0 || j > 0 || k > 0) ? 1u : 0u);
            }
          }
        }
        mma_commit(&empty[s]);
      }
      mma_commit(accum);
    }
  } else {
    // ---- epilogue: warps 2..5, thread <-> TMEM lane (row of the tile)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    mbar_wait(accum, 0, wc);
    tc_fence_after();
    // with an independent X the main loop ran alongside the previous kernel;
    // the epilogue reads its tables and writes what it may still read
    if (args.x_independent) griddep_wait();
    named_bar_sync(1, 128);            // every epilogue thread sees the same abort decision
    if (!*abort_flag) {
      const Epi& e = args.epi[seg];
      const int tile_id = mt + gridDim.x * nt;
      if (args.cluster_k > 1) {
        // split-K inside a cluster: this split's partial tile goes to the idle
        // pipeline buffers, [BN/4 column groups][128 rows][4]; the reduction
        // after the cluster barrier below reads it from every CTA
        float4* my = reinterpret_cast<float4*>(sA);
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
          float v[16];
          tmem_ld16(trow + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            my[((c >> 2) + q) * 128 + row] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      } else if (args.splits > 1) {
        // split-K: store this split's partial tile ([BN/4 column groups][128 rows][4],
        // so a warp moves 512 contiguous bytes per float4); gemm_splitk_epilogue_kernel
        // sums the splits in order and applies the epilogue
        float4* my = reinterpret_cast<float4*>(args.partials + (static_cast<long long>(tile_id) * args.splits + split) * (BN * 128));
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
          float v[16];
          tmem_ld16(trow + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            my[((c >> 2) + q) * 128 + row] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      } else {
        // the pipeline stages are idle now (every MMA retired): they hold the
        // staging tile, kStageCols token columns at a time
        uint8_t* stage = sA;
        constexpr int kCh = L::kStageCols;
#pragma unroll 1
        for (int t = 0; t < MT; ++t) {
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += kCh) {
#pragma unroll 1
            for (int c = c0; c < c0 + kCh; c += 16) {
              float v[16];
              tmem_ld16(trow + t * BN + c, v);
              tmem_wait_ld();
              epi_stage<16>(e, nt * BN + c, args.N, v, stage, c - c0, row);
            }
            named_bar_sync(1, 128);
            epi_flush(e, args.tok, m0 + t * 128, args.seg_rows[seg], nt * BN + c0, kCh, args.N, head, stage,
                      threadIdx.x - 64, 128, args.status);
            if (t + 1 < MT || c0 + kCh < BN) named_bar_sync(1, 128);  // the staging tile is refilled
          }
        }
      }
    }
  }
  // The producer and MMA warps arrive here with their elected lane last: the
  // warp must be reconverged before the CTA barrier (bar.sync is warp-aligned;
  // a warp that arrives split can release the barrier before the epilogue
  // warps arrive, and TMEM would be freed under their loads).
  __syncwarp();
  __syncthreads();
  if (args.cluster_k > 1) {
    // ---- split-K reduction across the cluster: CTA z of the S splits sums
    // rows [z 128/S, (z+1) 128/S) of the tile over all S partials, in split
    // order, and runs the epilogue on them.  Every CTA takes both barriers,
    // aborted or not, so none waits for a CTA that left.
    cluster_sync();  // every partial tile is in its CTA's shared memory
    if (warp >= 2 && !*abort_flag) {
      const int S = args.cluster_k;
      const int z = static_cast<int>(cluster_ctarank());
      const int nr = 128 / S, r0 = z * nr;
      const int tid = threadIdx.x - 64;
      const Epi& e = args.epi[seg];
      uint8_t* stage = sA + BN * 128 * 4;  // after the partial tile
      const uint32_t part = smem_u32(sA);
      for (int u = tid; u < (BN / 4) * nr; u += 128) {
        const int cg = u / nr, row = r0 + u % nr;
        // all S loads in flight together, then the sum in split order
        float4 p[kMaxClusterK];
#pragma unroll
        for (int q = 0; q < kMaxClusterK; ++q)
          if (q < S) p[q] = ld_shared_cluster_v4(mapa(part + (cg * 128 + row) * 16, static_cast<uint32_t>(q)));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < kMaxClusterK; ++q)
          if (q < S) {
            acc.x += p[q].x;
            acc.y += p[q].y;
            acc.z += p[q].z;
            acc.w += p[q].w;
          }
        const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
        epi_stage<4>(e, nt * BN + 4 * cg, args.N, vals, stage, 4 * cg, row);
      }
      named_bar_sync(1, 128);
      epi_flush(e, args.tok, m0, args.seg_rows[seg], nt * BN, BN, args.N, head, stage, tid, 128, args.status, r0,
                r0 + nr);
    }
    cluster_sync();  // no CTA reads another's shared memory any more
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Sums the split-K partials of every output tile in split order and applies
// the epilogue.  Grid (output tiles, BN/4): block x owns tile x, block y a
// group of 4 columns; thread = row of the tile (so the rotary partner row is a
// lane shuffle away).  All splits' loads of a thread are independent, so they
// are in flight together.
template <int BN>
__global__ void __launch_bounds__(128) gemm_splitk_epilogue_kernel(const __grid_constant__ GemmArgs args) {
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
  const int mt = blockIdx.x, cg = blockIdx.y, row = threadIdx.x;
  int seg = 0, head = 0, m0;
  if (args.mode == GEMM_DENSE) {
    while (seg + 1 < args.nseg && mt >= args.seg_tile0[seg + 1]) ++seg;
    m0 = (mt - args.seg_tile0[seg]) * 128;
  } else {
    const int tph = args.seg_tile0[1];
    head = mt / tph;
    m0 = (mt % tph) * 128;
  }
  const float4* p = reinterpret_cast<const float4*>(args.partials + static_cast<long long>(mt) * args.splits * (BN * 128)) +
                    cg * 128 + row;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
  for (int s = 0; s < args.splits; ++s) {
    const float4 t = __ldcg(p + static_cast<long long>(s) * (BN * 32));
    acc.x += t.x;
    acc.y += t.y;
    acc.z += t.z;
    acc.w += t.w;
  }
  __shared__ __align__(16) uint8_t stage[4 * 128 * 4];
  const Epi& e = args.epi[seg];
  const float v[4] = {acc.x, acc.y, acc.z, acc.w};
  epi_stage<4>(e, cg * 4, args.N, v, stage, 0, row);
  __syncthreads();
  epi_flush(e, args.tok, m0, args.seg_rows[seg], cg * 4, 4, args.N, head, stage, threadIdx.x, 128, args.status);
}

}  // namespace mla
