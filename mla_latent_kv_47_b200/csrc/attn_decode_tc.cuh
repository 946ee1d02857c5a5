// attn_decode_tc.cuh -- tensor-core split-KV decode attention over the MLA
// latent cache ("DeepSeek-V2 summary" (7shi.hateblo.jp), App. C with the
// absorption of its last paragraph): for each sequence b and head i,
//
//   s_ij = Q_lat[b,i] . [c^KV_j ; k^R_j]   (Q_lat pre-scaled by log2(e)/sqrt(d_h+d_R))
//   O_i  = sum_j 2^(s_ij - m_i) c^KV_j,   l_i = sum_j 2^(s_ij - m_i)
//
// over the rows j of a piece (a run of 64-token tiles of one sequence, as cut
// by the device planner), for d_c = 512, d_R = 64 and n_h <= 128 (fewer heads
// leave the spare MMA rows zero).
//
// Layout on the GPU.  All 128 heads of a sequence share each cache tile, so a
// tile is read from HBM once per sequence, not once per head.  The fp32 latent
// accumulator O (128 heads x 512) fills a whole SM's tensor memory, so each
// worker is a cluster of two CTAs that split the 576 latent columns:
//   CTA 0: columns c[0,256) and k^R (5 chunks of 64), O columns [0,256)
//   CTA 1: columns c[256,512)        (4 chunks),     O columns [256,512)
// Each CTA TMA-loads only its own columns of a tile, so the pair reads every
// cache byte exactly once.  Each computes a partial score S_r = Q_r C_r^T
// (tcgen05.mma, M = 128 heads, N = 64 tokens, Q_r held in TMEM), sends it to
// its partner through distributed shared memory as fp16, and forms
// S = fp16(S_0) + fp16(S_1): both CTAs round both halves the same way, so
// their softmax, P and running max are bit-identical.  The online softmax runs
// one thread per head (no cross-thread reductions) with a lazily refreshed
// max: O is rescaled only when a tile's max exceeds the running one by more
// than 2^8.  P (bf16) goes to shared memory and O_r += P C_r (N = 256, the
// same cache tile read as an MN-major operand) accumulates in TMEM.
//
// Warp roles (192 threads per CTA): warp 0 TMA, warp 1 TMEM owner and MMA
// issuer, warps 2-5 softmax / epilogue (thread = head = TMEM lane).
#pragma once
#include "mla.h"
#include "ptx.cuh"
#include "simt.cuh"

namespace mla {

constexpr int kAttnTileTokens = 64;
constexpr bool kAttnTcReady = true;

namespace attn {
constexpr int kStages = 4;
constexpr int kChunkBytes = 64 * 128;             // 64 token rows x 64 latent columns, bf16
constexpr int kStageBytes = 5 * kChunkBytes;      // up to 5 chunks per CTA
constexpr int kPBytes = 128 * 128;                // P: 128 heads x 64 tokens, bf16
constexpr int kXBytes = 128 * 128;                // partner's partial S: 128 heads x 64 tokens, fp16 (x2 buffers)
constexpr int kBarBytes = 256;
constexpr int kSmem = 1024 + kStages * kStageBytes + kPBytes + 2 * kXBytes + kBarBytes;
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemQ = 320, kTmemCols = 512;
constexpr float kRescaleLog2 = 8.f;
constexpr int kRow = 576;                         // d_c + d_R
}  // namespace attn

struct AttnArgs {
  CUtensorMap map_cache;       // cache rows [n_rows x 576] bf16, box {64 columns, 64 rows}, 128B swizzle
  const __nv_bfloat16* qlat;   // [B][n_h][576]
  const int64_t* seq_start;
  const int32_t* seqlen;
  const int* tile_start;
  const int* seg_start;
  int B, W, n_h;
  float* o_part;               // [slots][n_h][512]
  float* ml_part;              // [slots][n_h][2]
  int* status;
};

__device__ __forceinline__ int attn_chunk_col(uint32_t rank, int ci) {
  return rank == 0 ? (ci < 4 ? ci * 64 : 512) : 256 + ci * 64;
}

// fp16 pair (lo in the low half), rounded to nearest and saturated to the
// largest finite fp16 so an extreme partial score cannot become inf.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float2 unpack_half2(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    attn_decode_tc_kernel(const __grid_constant__ AttnArgs a) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* stages = smem;
  uint8_t* pbuf = stages + kStages * kStageBytes;
  uint8_t* xbuf = pbuf + kPBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(xbuf + 2 * kXBytes);
  uint64_t* empty = full + kStages;
  uint64_t* s_full = empty + kStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;
  uint64_t* p_free = p_full + 1;
  uint64_t* x_full = p_free + 1;   // [2]
  uint64_t* x_free = x_full + 2;   // [2]
  uint64_t* q_full = x_free + 2;
  uint64_t* o_done = q_full + 1;
  uint64_t* drain = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int w = blockIdx.x >> 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = rank == 0 ? 5 : 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&x_full[i], 4);  // one arrival per softmax warp of the partner
      mbar_init(&x_free[i], 4);
    }
    mbar_init(q_full, 128);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&a.map_cache);
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  cluster_sync();  // the partner's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // Q_lat and the new cache rows come from the preceding kernels
  WaitCtx wc{a.status, abort_flag};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
        if (*abort_flag) return;
        const long long row0 = a.seq_start[p.b];
        for (int t = p.t0; t < p.t1; ++t, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, wc)) return;
          mbar_arrive_expect_tx(&full[s], nchunks * kChunkBytes);
          uint8_t* dst = stages + s * kStageBytes;
          const int y = static_cast<int>(row0 + static_cast<long long>(t) * 64);
          for (int ci = 0; ci < nchunks; ++ci)
            tma_load_2d(dst + ci * kChunkBytes, &a.map_cache, &full[s], attn_chunk_col(rank, ci), y, pol);
        }
      });
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 64, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 256, false, true);
      int it = 0, piece = 0;
      for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
        if (*abort_flag) return;
        if (!mbar_wait(q_full, piece & 1, wc)) return;
        tc_fence_after();
        const int nt = p.t1 - p.t0;
        // Event-driven issue: S(j) as soon as its tile landed and S(j-1) was read
        // out (the softmax reads S one tile ahead), PV(j) as soon as P(j) is
        // written; S first, so the softmax never waits behind a PV.
        int ns = 0, npv = 0;
        uint64_t t_idle = globaltimer();
        while (npv < nt) {
          bool issued = false;
          if (ns < nt) {
            const int g = it + ns;
            const int s = g % kStages;
            if (mbar_try_wait(smem_u32(&full[s]), (g / kStages) & 1) && mbar_try_wait(smem_u32(s_free), (g & 1) ^ 1)) {
              tc_fence_after();
              const uint32_t st = smem_u32(stages + s * kStageBytes);
              for (int ci = 0; ci < nchunks; ++ci) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  mma_ts(tmem + kTmemS, tmem + kTmemQ + ci * 32 + kk * 8,
                         sdesc_sw128(st + ci * kChunkBytes + kk * 32, 16, 1024), idesc_s, (ci | kk) ? 1u : 0u);
                }
              }
              mma_commit(s_full);
              ++ns;
              issued = true;
            }
          }
          if (!issued && npv < ns) {
            const int g = it + npv;
            const int s = g % kStages;
            if (mbar_try_wait(smem_u32(p_full), g & 1)) {
              tc_fence_after();
              const uint32_t st = smem_u32(stages + s * kStageBytes);
              const uint32_t pb = smem_u32(pbuf);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                mma_ss(tmem + kTmemO, sdesc_sw128(pb + kk * 32, 16, 1024), sdesc_sw128(st + kk * 2048, 8192, 1024),
                       idesc_pv, (npv > 0 || kk > 0) ? 1u : 0u);
              }
              mma_commit(p_free);
              mma_commit(&empty[s]);
              if (npv == nt - 1) mma_commit(o_done);
              ++npv;
              issued = true;
            }
          }
          if (issued) {
            t_idle = globaltimer();
          } else if (*abort_flag) {
            return;
          } else if (globaltimer() - t_idle > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(a.status, FAULT_WAIT_TIMEOUT);
            return;
          }
        }
        it += nt;
        ++piece;
      });
      mma_commit(drain);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp & 3;
    const int h = q4 * 32 + lane;  // head = TMEM lane
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t x_row = smem_u32(xbuf) + h * 128;
    const uint32_t x_row_peer = mapa(smem_u32(xbuf), peer) + h * 128;
    const uint32_t xfull_peer = mapa(smem_u32(x_full), peer);
    const uint32_t xfree_peer = mapa(smem_u32(x_free), peer);
    const uint32_t p_row = smem_u32(pbuf) + h * 128;
    const int sw = h & 7;
    // Partial scores of global tile g: read from TMEM, rounded to fp16 into
    // `out`, and sent to the partner's exchange buffer g & 1.  The partner is
    // told once per warp (after the warp's stores, ordered by the warp barrier).
    auto send = [&](int g, uint32_t (&out)[32]) -> bool {
      if (!mbar_wait(s_full, g & 1, wc)) return false;
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tl + kTmemS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tl + kTmemS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_free);
#pragma unroll
      for (int j = 0; j < 32; ++j) out[j] = pack_half2(__uint_as_float(sr[2 * j]), __uint_as_float(sr[2 * j + 1]));
      const int slot = g & 1;
      if (!mbar_wait<true>(&x_free[slot], ((g >> 1) & 1) ^ 1, wc)) return false;
      const uint32_t dst = x_row_peer + slot * kXBytes;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        st_cluster_v4(dst + ((i ^ sw) << 4), make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]));
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(xfull_peer + slot * 8);
      return true;
    };
    int it = 0, piece = 0;
    for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
      if (*abort_flag) return;
      // ---- this CTA's half of Q_lat[b, h] into TMEM (MMA A operand)
      const bool head = h < a.n_h;
      const __nv_bfloat16* qrow = a.qlat + (static_cast<long long>(p.b) * a.n_h + (head ? h : 0)) * kRow;
      for (int ci = 0; ci < nchunks; ++ci) {
        const uint4* src = reinterpret_cast<const uint4*>(qrow + attn_chunk_col(rank, ci));
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = head ? src[i] : make_uint4(0, 0, 0, 0);
          r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
        }
        tmem_st32(tl + kTmemQ + ci * 32, r);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(q_full);

      const int L1 = a.seqlen[p.b] + 1;
      float m_run = -INFINITY, l_run = 0.f;
      const int nt = p.t1 - p.t0;
      uint32_t mine[32];
      if (nt > 0 && !send(it, mine)) return;
      for (int k = 0; k < nt; ++k) {
        const int g = it + k;
        const int t = p.t0 + k;
        // the next tile's partial goes out before this tile's partner half is awaited,
        // so the exchange latency overlaps the softmax of this tile
        uint32_t nxt[32];
        if (k + 1 < nt && !send(g + 1, nxt)) return;
        const int slot = g & 1;
        if (!mbar_wait<true>(&x_full[slot], (g >> 1) & 1, wc)) return;
        uint32_t theirs[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = ld_shared_v4(x_row + slot * kXBytes + ((i ^ sw) << 4));
          theirs[4 * i] = v.x; theirs[4 * i + 1] = v.y; theirs[4 * i + 2] = v.z; theirs[4 * i + 3] = v.w;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(xfree_peer + slot * 8);
        // ---- full scores (same bits in both CTAs), masked beyond the sequence
        const int valid = min(64, L1 - t * 64);
        float mt = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float2 x = unpack_half2(mine[j]), y = unpack_half2(theirs[j]);
          const float s0 = (2 * j < valid) ? x.x + y.x : -INFINITY;
          const float s1 = (2 * j + 1 < valid) ? x.y + y.y : -INFINITY;
          mt = fmaxf(mt, fmaxf(s0, s1));
        }
        float m_new = m_run, alpha = 1.f;
        bool rescale = false;
        if (k == 0) {
          m_new = mt;
        } else if (mt > m_run + kRescaleLog2) {
          m_new = mt;
          alpha = ex2_approx(m_run - m_new);
          rescale = true;
        }
        uint32_t pk[32];
        float lsum = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float2 x = unpack_half2(mine[j]), y = unpack_half2(theirs[j]);
          const float s0 = (2 * j < valid) ? x.x + y.x : -INFINITY;
          const float s1 = (2 * j + 1 < valid) ? x.y + y.y : -INFINITY;
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(ex2_approx(s0 - m_new), ex2_approx(s1 - m_new));
          const float2 f = __bfloat1622float2(b2);
          lsum += f.x + f.y;
          pk[j] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        l_run = l_run * alpha + lsum;
        m_run = m_new;
        // ---- previous PV done: P buffer free, O settled
        if (!mbar_wait(p_free, (g & 1) ^ 1, wc)) return;
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
          for (int c = 0; c < 256; c += 32) {
            uint32_t o[32];
            tmem_ld32(tl + kTmemO + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tl + kTmemO + c, o);
          }
          tmem_wait_st();
        }
        if (valid < 64) {
          // rows past the sequence may hold anything (even NaN); 0 * NaN would
          // poison O, so the rows this CTA multiplies into O are zeroed
          uint8_t* st = stages + (g % kStages) * kStageBytes;
          const int n16 = (64 - valid) * 32;
          for (int idx = h; idx < n16; idx += 128) {
            const int row = valid + (idx >> 5), c16 = idx & 31;
            *reinterpret_cast<uint4*>(st + (c16 >> 3) * kChunkBytes + row * 128 + (c16 & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
          st_shared_v4(p_row + ((i ^ sw) << 4), make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]));
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
        if (k + 1 < nt) {
#pragma unroll
          for (int j = 0; j < 32; ++j) mine[j] = nxt[j];
        }
      }
      // ---- epilogue of the piece: unnormalised O_r, m, l
      if (!mbar_wait(o_done, piece & 1, wc)) return;
      tc_fence_after();
      float* dst = a.o_part + (static_cast<long long>(p.slot) * a.n_h + h) * 512 + rank * 256;
      for (int c = 0; c < 256; c += 32) {
        uint32_t o[32];
        tmem_ld32(tl + kTmemO + c, o);
        tmem_wait_ld();
        if (head) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(dst + c)[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                                                __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
        }
      }
      if (rank == 0 && head) {
        a.ml_part[(static_cast<long long>(p.slot) * a.n_h + h) * 2] = m_run;
        a.ml_part[(static_cast<long long>(p.slot) * a.n_h + h) * 2 + 1] = l_run;
      }
      tc_fence_before();
      it += nt;
      ++piece;
    });
  }
  // ---- teardown: every MMA retired, the partner no longer writes into this CTA.
  // The next kernel is released only now: its CTAs would otherwise sit on
  // these SMs during the main loop.
  if (threadIdx.x == 0) griddep_launch_dependents();
  if (warp == 1) {
    __syncwarp();
    if (lane == 0) {  // bounded, and not cut short by an abort: TMEM is freed only after the MMAs retire
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(smem_u32(drain), 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  }
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mla
