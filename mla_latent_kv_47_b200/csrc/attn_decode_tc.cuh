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
// (tcgen05.mma, M = 128 heads, N = 64 tokens, into one of two TMEM buffers;
// the c^KV part of Q_r in TMEM, CTA 0's k^R part in shared memory) and both CTAs
// form S = fp16(S_0) + fp16(S_1) from the same rounded halves, so their
// softmax, P and running max are bit-identical.  O_r += P C_r (N = 256, the
// same cache tile read as an MN-major operand) accumulates in TMEM.
//
// Warp roles (448 threads per CTA); each tile flows through them in order:
//   warp 0      TMA producer (4-stage ring of tiles)
//   warp 1      TMEM owner and MMA issuer: S(j) as soon as tile j landed and
//               the S buffer of tile j-2 was read out, PV as soon as P is written
//   warps 2-5   exchange: read S from TMEM, round it to fp16, push it into the
//               partner's shared memory with st.async (its bytes complete the
//               partner's barrier, so the sender neither fences nor waits) and
//               write this CTA's rounded half back over the S buffer for the
//               softmax (the S buffer is freed once the softmax read it).  The
//               partner hands a slot back the same way: a 4-byte st.async per
//               softmax warp that completes this CTA's slot-free barrier.
//   warps 6-13  softmax: warp 6+i and warp 10+i share lane quarter i mod 4,
//               16 heads each; two threads per head (tokens 0-31 and 32-63 of
//               the tile, via the 16-lane TMEM access shape), so a head's tile
//               max is one shuffle.  Online softmax with a lazily refreshed
//               max (O is rescaled only when a tile's max exceeds the running
//               one by more than 2^8), P (bf16) into shared memory, and the
//               per-piece epilogue.
// The exchange warps use thread = head = TMEM lane (warp w owns lanes
// 32 (w mod 4) ..).
#pragma once
#include "mla.h"
#include "ptx.cuh"
#include "simt.cuh"

namespace mla {

constexpr int kAttnTileTokens = 64;
constexpr bool kAttnTcReady = true;

namespace attn {
constexpr int kStages = 4;
constexpr int kThreads = 448;
constexpr int kChunkBytes = 64 * 128;             // 64 token rows x 64 latent columns, bf16
constexpr int kStageBytes = 5 * kChunkBytes;      // up to 5 chunks per CTA
constexpr int kXBytes = 128 * 128;                // one half of S: 128 heads x 64 tokens, fp16
constexpr int kPBytes = 128 * 128;                // P: 128 heads x 64 tokens, bf16
constexpr int kXSlots = 2;                        // exchange slots for the partner's score half
constexpr int kPBufs = 1;                         // P buffers
constexpr int kQRBytes = 128 * 128;               // CTA 0's k^R part of Q: 128 heads x 64, bf16 (MMA A operand)
constexpr int kBarBytes = 512;
// stages | partner's S half x kXSlots | P x kPBufs | k^R part of Q | barriers
constexpr int kSmem = 1024 + kStages * kStageBytes + kXSlots * kXBytes + kPBufs * kPBytes + kQRBytes + kBarBytes;
// TMEM columns: O half [0,256), S buffers [256,320) and [320,384) (after the
// exchange, their first 32 columns hold this CTA's fp16-rounded half), c^KV
// part of the Q half (bf16 pairs) [384,512)
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemQ = 384, kTmemCols = 512;
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(attn::kThreads, 1)
    attn_decode_tc_kernel(const __grid_constant__ AttnArgs a) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* stages = smem;
  uint8_t* xpeer = stages + kStages * kStageBytes;  // [kXSlots] the partner's half of S (fp16), written by the partner
  uint8_t* pbuf = xpeer + kXSlots * kXBytes;        // [kPBufs] P (bf16), MMA A operand
  uint8_t* qr = pbuf + kPBufs * kPBytes;            // CTA 0: k^R part of Q (bf16), MMA A operand
  uint64_t* full = reinterpret_cast<uint64_t*>(qr + kQRBytes);
  uint64_t* empty = full + kStages;
  uint64_t* s_full = empty + kStages;  // [2] S(j) in buffer j & 1 (MMA -> exchange)
  uint64_t* s_free = s_full + 2;       // [2] buffer read out by the softmax (softmax -> MMA)
  uint64_t* xo_full = s_free + 2;      // [2] own rounded half written back (exchange -> softmax)
  uint64_t* x_full = xo_full + 2;    // [kXSlots] partner's half landed (st.async bytes)
  uint64_t* x_free = x_full + kXSlots;  // [kXSlots] partner's half consumed (signals from the partner's softmax)
  uint64_t* p_full = x_free + kXSlots;  // [kPBufs]
  uint64_t* p_free = p_full + kPBufs;   // [kPBufs]
  uint64_t* q_full = p_free + kPBufs;
  uint64_t* o_done = q_full + 1;
  uint64_t* drain = o_done + 1;
  uint32_t* sig = reinterpret_cast<uint32_t*>(drain + 1);  // [kXSlots][8] landing words of the partner's slot-free signals
  uint32_t* tmem_slot = sig + 8 * kXSlots;
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 8);   // one arrival per softmax warp
      mbar_init(&xo_full[i], 4);  // one arrival per exchange warp
    }
    for (int i = 0; i < kXSlots; ++i) {
      mbar_init(&x_full[i], 1);   // armed once per phase with the expected bytes
      mbar_init(&x_free[i], 1);   // armed by the exchange before each use; 8 x 4 signal bytes from the partner
    }
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(&p_full[i], 8);   // one arrival per softmax warp
      mbar_init(&p_free[i], 1);
    }
    mbar_init(q_full, 128);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    // phase 0 of every exchange slot expects the partner's 16 KB
    for (int i = 0; i < kXSlots; ++i) mbar_arrive_expect_tx(&x_full[i], kXBytes);
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&a.map_cache);
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  cluster_sync();  // the partner's barriers exist (and are armed) before any remote access
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
        // PV first: it gates the softmax of the next tile, while S only has
        // to be ready by the time the exchange warps come back for it.
        int ns = 0, npv = 0;
        uint32_t spins = 0;
        uint64_t t_idle = 0;
        while (npv < nt) {
          bool issued = false;
          if (npv < ns) {
            const int g = it + npv;
            const int s = g % kStages;
            const int b = g % kPBufs;
            if (mbar_test_wait(smem_u32(&p_full[b]), (g / kPBufs) & 1)) {
              tc_fence_after();
              const uint32_t st = smem_u32(stages + s * kStageBytes);
              const uint32_t pb = smem_u32(pbuf + b * kPBytes);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                mma_ss(tmem + kTmemO, sdesc_sw128(pb + kk * 32, 16, 1024), sdesc_sw128(st + kk * 2048, 8192, 1024),
                       idesc_pv, (npv > 0 || kk > 0) ? 1u : 0u);
              }
              mma_commit(&p_free[b]);
              mma_commit(&empty[s]);
              if (npv == nt - 1) mma_commit(o_done);
              ++npv;
              issued = true;
            }
          }
          if (!issued && ns < nt) {
            const int g = it + ns;
            const int s = g % kStages;
            const int sb = g & 1;
            if (mbar_test_wait(smem_u32(&full[s]), (g / kStages) & 1) &&
                mbar_test_wait(smem_u32(&s_free[sb]), ((g >> 1) & 1) ^ 1)) {
              tc_fence_after();
              const uint32_t st = smem_u32(stages + s * kStageBytes);
              const uint32_t dS = tmem + kTmemS + sb * 64;
              for (int ci = 0; ci < 4; ++ci) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  mma_ts(dS, tmem + kTmemQ + ci * 32 + kk * 8, sdesc_sw128(st + ci * kChunkBytes + kk * 32, 16, 1024),
                         idesc_s, (ci | kk) ? 1u : 0u);
                }
              }
              if (nchunks == 5) {  // CTA 0: the k^R chunk, Q_R from shared memory
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  mma_ss(dS, sdesc_sw128(smem_u32(qr) + kk * 32, 16, 1024),
                         sdesc_sw128(st + 4 * kChunkBytes + kk * 32, 16, 1024), idesc_s, 1u);
                }
              }
              mma_commit(&s_full[sb]);
              ++ns;
              issued = true;
            }
          }
          // idle bookkeeping every 256 empty polls: abort, and the wait limit
          if (issued) {
            spins = 0;
          } else if ((++spins & 255u) == 0) {
            if (*abort_flag) return;
            const uint64_t now = globaltimer();
            if (spins == 256) {
              t_idle = now;
            } else if (now - t_idle > kWaitLimitNs) {
              *abort_flag = 1;
              atomicOr(a.status, FAULT_WAIT_TIMEOUT);
              return;
            }
          }
        }
        it += nt;
        ++piece;
      });
      mma_commit(drain);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ exchange
    const int q4 = warp & 3;
    const int h = q4 * 32 + lane;  // head = TMEM lane
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int sw = h & 7;
    const uint32_t peer_row = mapa(smem_u32(xpeer), peer) + h * 128;
    const uint32_t xfull_peer = mapa(smem_u32(x_full), peer);
    const uint32_t qr_row = smem_u32(qr) + h * 128;
    const bool arm = warp == 2 && lane == 0;
    int it = 0;
    for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
      if (*abort_flag) return;
      // ---- this CTA's half of Q_lat[b, h] into TMEM (MMA A operand).  The
      // previous piece's last S has been read out, so no MMA still reads Q.
      const bool head = h < a.n_h;
      const __nv_bfloat16* qrow = a.qlat + (static_cast<long long>(p.b) * a.n_h + (head ? h : 0)) * kRow;
      for (int ci = 0; ci < 4; ++ci) {
        const uint4* src = reinterpret_cast<const uint4*>(qrow + attn_chunk_col(rank, ci));
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = head ? src[i] : make_uint4(0, 0, 0, 0);
          r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
        }
        tmem_st32(tl + kTmemQ + ci * 32, r);
      }
      if (nchunks == 5) {  // CTA 0: the k^R part of Q into shared memory, 128-byte swizzled rows
        const uint4* src = reinterpret_cast<const uint4*>(qrow + attn_chunk_col(rank, 4));
#pragma unroll
        for (int i = 0; i < 8; ++i) st_shared_v4(qr_row + ((i ^ sw) << 4), head ? src[i] : make_uint4(0, 0, 0, 0));
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(q_full);

      const int nt = p.t1 - p.t0;
      for (int k = 0; k < nt; ++k) {
        const int g = it + k;
        const int slot = g % kXSlots;
        const uint32_t ph = (g / kXSlots) & 1;
        const int sb = g & 1;
        if (!mbar_wait(&s_full[sb], (g >> 1) & 1, wc)) return;
        tc_fence_after();
        uint32_t hx[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t sr[32];
          tmem_ld32(tl + kTmemS + sb * 64 + half * 32, sr);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            hx[half * 16 + j] = pack_half2(__uint_as_float(sr[2 * j]), __uint_as_float(sr[2 * j + 1]));
        }
        // partner first: its copy has the longer way to go
        if (!mbar_wait<true>(&x_free[slot], ph ^ 1, wc)) return;
        // the partner returns this use of the slot with 8 signals of 4 bytes;
        // armed before this warp's data goes out, so no signal can precede it
        if (arm) mbar_arrive_expect_tx(&x_free[slot], 32);
        const uint32_t dst = peer_row + slot * kXBytes;
        const uint32_t bar = xfull_peer + slot * 8;  // x_full[slot] in the partner
#pragma unroll
        for (int i = 0; i < 8; ++i)
          st_async_v4(dst + ((i ^ sw) << 4), make_uint4(hx[4 * i], hx[4 * i + 1], hx[4 * i + 2], hx[4 * i + 3]), bar);
        // own rounded half over the first 32 columns of the S buffer
        tmem_st32(tl + kTmemS + sb * 64, hx);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&xo_full[sb]);
      }
      it += nt;
    });
    // The partner's signals for the last use of each slot land in this CTA's
    // shared memory: they must have arrived before the CTA may exit.
    if (arm && !*abort_flag) {
      for (int s2 = 0; s2 < kXSlots; ++s2) {
        const int uses = (it + kXSlots - 1 - s2) / kXSlots;  // tiles g < it with g % kXSlots == s2
        if (uses > 0 && !mbar_wait<true>(&x_free[s2], (uses - 1) & 1, wc)) break;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp & 3;
    const int hs = (warp - 6) >> 2;  // which 16 heads of the lane quarter
    const int th = lane >> 4;        // token half of the tile: [32 th, 32 th + 32)
    const int h = q4 * 32 + hs * 16 + (lane & 15);
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32 + hs * 16) << 16);
    const int sw = h & 7;
    const bool leader = warp == 6;   // re-arms the exchange barriers
    const uint32_t peer_row = smem_u32(xpeer) + h * 128;
    const uint32_t p_row = smem_u32(pbuf) + h * 128;
    const uint32_t xfree_peer = mapa(smem_u32(x_free), peer);
    const uint32_t sig_peer = mapa(smem_u32(sig), peer) + (warp - 6) * 4;
    int it = 0, piece = 0;
    for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
      if (*abort_flag) return;
      const bool head = h < a.n_h;
      const int L1 = a.seqlen[p.b] + 1;
      float m_run = -INFINITY, l_run = 0.f;  // l_run: this thread's token half only
      const int nt = p.t1 - p.t0;
      for (int k = 0; k < nt; ++k) {
        const int g = it + k;
        const int t = p.t0 + k;
        const int slot = g % kXSlots;
        const uint32_t ph = (g / kXSlots) & 1;
        const int sb = g & 1;
        if (!mbar_wait(&xo_full[sb], (g >> 1) & 1, wc)) return;
        if (!mbar_wait<true>(&x_full[slot], ph, wc)) return;
        tc_fence_after();
        // ---- full scores of this thread's 32 tokens (same bits in both CTAs)
        uint32_t own[16];
        tmem_ld16x2(tl + kTmemS + sb * 64, own);
        uint4 pv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) pv[i] = ld_shared_v4(peer_row + slot * kXBytes + (((th * 4 + i) ^ sw) << 4));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s_free[sb]);  // S buffer sb may take S(g + 2)
          // the slot's next phase expects the partner's next 16 KB; armed
          // before the slot is released, so no byte can land ahead of it
          if (leader) mbar_arrive_expect_tx(&x_full[slot], kXBytes);
        }
        const int valid = min(64, L1 - t * 64) - th * 32;  // valid tokens of this half (may be <= 0)
        float sc[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t vv[4] = {pv[i].x, pv[i].y, pv[i].z, pv[i].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x = unpack_half2(own[4 * i + e]), y = unpack_half2(vv[e]);
            sc[8 * i + 2 * e] = x.x + y.x;
            sc[8 * i + 2 * e + 1] = x.y + y.y;
          }
        }
        // every value read from the partner's half is consumed: hand the slot back
        __syncwarp();
        if (lane == 0) st_async_b32(sig_peer + slot * 32, 0u, xfree_peer + slot * 8);  // into sig[slot][warp - 6]
        if (__any_sync(0xffffffffu, valid < 32)) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j >= valid) sc[j] = -INFINITY;
        }
        float mh = sc[0];
#pragma unroll
        for (int j = 1; j < 32; ++j) mh = fmaxf(mh, sc[j]);
        const float mt = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, 16));  // the head's other token half
        float m_new = m_run, alpha = 1.f;
        bool rescale = false;
        if (k == 0) {
          m_new = mt;
        } else if (mt > m_run + kRescaleLog2) {
          m_new = mt;
          alpha = ex2_approx(m_run - m_new);
          rescale = true;
        }
        uint32_t pk[16];
        float lsum = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float p0 = ex2_approx(sc[2 * j] - m_new), p1 = ex2_approx(sc[2 * j + 1] - m_new);
          lsum += p0 + p1;
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          pk[j] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        l_run = l_run * alpha + lsum;
        m_run = m_new;
        // ---- P buffer b is free once PV(g-2) retired
        const int b = g % kPBufs;
        if (!mbar_wait(&p_free[b], ((g / kPBufs) & 1) ^ 1, wc)) return;
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
          // O must hold PV(g-1) before it is scaled (k >= 1 here, so g >= 1)
          if (kPBufs > 1 && !mbar_wait(&p_free[(g - 1) % kPBufs], ((g - 1) / kPBufs) & 1, wc)) return;
          tc_fence_after();
          for (int c = 0; c < 256; c += 32) {
            uint32_t o[16];
            tmem_ld16x2(tl + kTmemO + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16x2(tl + kTmemO + c, o);
          }
          tmem_wait_st();
        }
        const int v64 = valid + th * 32;
        if (v64 < 64) {
          // rows past the sequence may hold anything (even NaN); 0 * NaN would
          // poison O, so the rows this CTA multiplies into O are zeroed
          uint8_t* st = stages + (g % kStages) * kStageBytes;
          const int n16 = (64 - v64) * 32;
          for (int idx = (warp - 6) * 32 + lane; idx < n16; idx += 256) {
            const int row = v64 + (idx >> 5), c16 = idx & 31;
            *reinterpret_cast<uint4*>(st + (c16 >> 3) * kChunkBytes + row * 128 + (c16 & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
          st_shared_v4(p_row + b * kPBytes + (((th * 4 + i) ^ sw) << 4),
                       make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]));
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
      }
      // ---- epilogue of the piece: unnormalised O_r, m, l
      if (!mbar_wait(o_done, piece & 1, wc)) return;
      tc_fence_after();
      float* dst = a.o_part + (static_cast<long long>(p.slot) * a.n_h + h) * 512 + rank * 256 + th * 16;
      for (int c = 0; c < 256; c += 32) {
        uint32_t o[16];
        tmem_ld16x2(tl + kTmemO + c, o);
        tmem_wait_ld();
        if (head) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            reinterpret_cast<float4*>(dst + c)[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                                                __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
        }
      }
      const float l_head = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
      if (rank == 0 && th == 0 && head) {
        a.ml_part[(static_cast<long long>(p.slot) * a.n_h + h) * 2] = m_run;
        a.ml_part[(static_cast<long long>(p.slot) * a.n_h + h) * 2 + 1] = l_head;
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
  __syncwarp();  // every warp reconverged (elected producer / issuer lanes) before the aligned barriers
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mla
