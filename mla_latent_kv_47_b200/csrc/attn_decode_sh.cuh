// attn_decode_sh.cuh -- tensor-core split-KV decode attention for few heads
// (n_h <= 16, e.g. DeepSeek-V2-Lite), bf16 latent cache rows.  It computes
// what attn_decode_tc.cuh computes ("DeepSeek-V2 summary" (7shi.hateblo.jp),
// App. C with the absorption of its last paragraph),
//
//   s_ij = Q_lat[b,i] . [c^KV_j ; k^R_j]   (Q_lat pre-scaled by log2(e)/sqrt(d_h+d_R))
//   O_i  = sum_j 2^(s_ij - m_i) c^KV_j,   l_i = sum_j 2^(s_ij - m_i)
//
// over the pieces the device planner cuts, and writes the same partials.
//
// With 16 heads, the head-major form (M = heads) would leave 7/8 of every
// M = 128 MMA empty.  Here the tokens are the M dimension instead:
//   S^T = C Q^T       tcgen05.mma M = 64 cached tokens, N = 16 heads, K = 576
//   O^T += C^T P^T    M = 128 latent columns (4 tiles), N = 16 heads, K = 64 tokens
// so one CTA (one SM) holds the whole accumulator, O^T: 512 x 16 fp32, in 64
// TMEM columns, and a worker is a single CTA: 148 workers, no pair exchange.
// The M = 64 score tile puts token 16 q + i in TMEM lane 32 q + i.
//
// The softmax reference is the pair kernel's: the max over a piece's first
// tile is the piece's m for each head, every P of the piece is 2^(s - m), O
// and l are never rescaled, and P is capped at 2^96 (FAULT_RANGE past it).
//
// Warp roles (192 threads): warp 0 TMA producer (2 stages of 64 tokens x 576
// columns), warp 1 TMEM owner and MMA issuer, warps 2-5 Q, the softmax (warp
// q takes tokens 16 q .. 16 q + 15 of a tile, two threads per token, 8 heads
// each) and the per-piece epilogue.  Q has two buffers: the next piece's Q is
// loaded as soon as the current piece's last P is written, so the next
// piece's score MMAs run during the epilogue, and the epilogue writes (m, l)
// before it waits for the last PV product.  A tile's 36 score MMAs are issued
// back to back once its whole stage has landed: issuing them a chunk at a
// time as the chunks land measured slower.
#pragma once
#include "attn_decode_tc.cuh"

namespace mla {
namespace attn_sh {
constexpr int kThreads = 192;
constexpr int kNH = 16;                               // heads (N of both products)
constexpr int kTile = 64;                             // tokens per tile
constexpr int kStages = 2;
constexpr int kChunk = kTile * 128;                   // 64 rows x 64 columns bf16, 128B swizzle
constexpr int kStageBytes = 9 * kChunk;               // c^KV chunks 0-7, k^R chunk 8
constexpr int kQChunk = kNH * 128;                    // 16 heads x 64 columns
constexpr int kQBytes = 9 * kQChunk;
constexpr int kPBytes = kNH * 128;                    // P^T: 16 heads x 64 tokens, bf16, 128B swizzle
constexpr int kAuxBytes = 2048;
// TMEM columns: S^T two buffers of 16 [0,32), O^T four tiles of 16 [32,96)
constexpr uint32_t kTmemS = 0, kTmemO = 32, kTmemCols = 128;
constexpr float kRangeLog2 = 96.f;
constexpr int kRow = 576;
constexpr int kSmem = 1024 + kStages * kStageBytes + 2 * kQBytes + 2 * kPBytes + kAuxBytes;
static_assert(kSmem <= 232448, "shared memory budget");
static_assert(kQChunk % 1024 == 0 && kPBytes % 1024 == 0, "1024-byte alignment of the swizzled tiles");
}  // namespace attn_sh

// 16 lanes x 32 bit, twice, 8 columns: thread t < 16 reads lane (taddr.lane +
// t), columns taddr.col .. +7; thread t >= 16 reads lane (taddr.lane + t -
// 16), columns taddr.col + 8 .. +15.
__device__ __forceinline__ void tmem_ld16x2_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], 8;"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

__global__ void __launch_bounds__(attn_sh::kThreads, 1) attn_decode_sh_kernel(const __grid_constant__ AttnArgs a) {
  using namespace attn_sh;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* stages = smem;
  uint8_t* qs = stages + kStages * kStageBytes;  // [2] Q: 9 chunks of 16 heads x 64 columns (MMA B operand)
  uint8_t* pbuf = qs + 2 * kQBytes;              // [2] P^T (MMA B operand)
  uint8_t* aux = pbuf + 2 * kPBytes;
  float* mxs = reinterpret_cast<float*>(aux);    // [2 pieces][4 warps][16 heads] maxima of the first tile
  float* lxs = mxs + 2 * 4 * kNH;                // [4 warps][16 heads] l of the piece
  uint64_t* full = reinterpret_cast<uint64_t*>(aux + 1024);
  uint64_t* empty = full + kStages;
  uint64_t* s_full = empty + kStages;   // [2] S^T(j) in TMEM buffer j % 2
  uint64_t* s_free = s_full + 2;        // [2] S^T(j) read out
  uint64_t* p_full = s_free + 2;        // [2] P^T(j) written (buffer j % 2)
  uint64_t* p_free = p_full + 2;        // [2] PV(j) retired
  uint64_t* q_full = p_free + 2;        // [2] Q of piece j in buffer j % 2
  uint64_t* q_free = q_full + 2;        // [2] last S of piece j retired
  uint64_t* o_done = q_free + 2;
  uint64_t* drain = o_done + 1;
  uint64_t* mx_bar = drain + 1;         // [2] the four warps' maxima of piece j in mxs (buffer j % 2)
  uint64_t* l_bar = mx_bar + 2;         // the four warps' l of the piece in lxs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(l_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert(1024 + (2 * kStages + 17) * 8 + 8 <= kAuxBytes, "aux layout");
  static_assert((2 * 4 * kNH + 4 * kNH) * 4 <= 1024, "aux layout: maxima and l");

  const int w = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);  // one arrival per softmax warp
      mbar_init(&p_full[i], 4);
      mbar_init(&p_free[i], 1);
      mbar_init(&mx_bar[i], 4);
      mbar_init(&q_full[i], 4);
      mbar_init(&q_free[i], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    mbar_init(l_bar, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&a.map_cache);
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // Q_lat and the new cache rows come from the preceding kernels
  WaitCtx wc{a.status, abort_flag};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      const uint64_t pol = policy_evict_first();  // every byte is read once
      int it = 0;
      for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
        if (*abort_flag) return;
        const long long row0 = a.lay.block_table ? 0 : a.lay.seq_start[p.b];  // contiguous layout
        for (int t = p.t0; t < p.t1; ++t, ++it) {
          // a tile lies within one page; a tile without a page (a capacity
          // fault of the call) loads rows past the tensor, which read as zero
          long long y0 = a.lay.block_table ? a.lay.row(p.b, static_cast<long long>(t) * kTile)
                                           : row0 + static_cast<long long>(t) * kTile;
          if (y0 < 0) y0 = a.n_rows;
          const int s = it % kStages;
          if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, wc)) return;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          uint8_t* dst = stages + s * kStageBytes;
          const int y = static_cast<int>(y0);
          for (int c = 0; c < 9; ++c) {
            tma_load_2d(dst + c * kChunk, &a.map_cache, &full[s], c * 64, y, pol);
            tma_load_2d(dst + c * kChunk + kChunk / 2, &a.map_cache, &full[s], c * 64, y + 32, pol);
          }
        }
      });
      drain_ring(full, kStages, it);  // every issued load has landed before the CTA may leave
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_bf16(64, kNH, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, kNH, true, false);
      int it = 0, piece = 0;
      for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
        if (*abort_flag) return;
        if (!mbar_wait(&q_full[piece & 1], (piece >> 1) & 1, wc)) return;
        tc_fence_after();
        const int nt = p.t1 - p.t0;
        int ns = 0, npv = 0;
        uint32_t spins = 0;
        uint64_t t_idle = 0;
        const uint32_t qb = smem_u32(qs + (piece & 1) * kQBytes);
        while (npv < nt) {
          bool issued = false;
          if (npv < ns) {  // O^T += C^T P^T(g)
            const int g = it + npv;
            const int s = g % kStages, b = g & 1;
            if (mbar_test_wait(smem_u32(&p_full[b]), (g >> 1) & 1)) {
              tc_fence_after();
              const uint32_t st = smem_u32(stages + s * kStageBytes);
              const uint32_t pb = smem_u32(pbuf + b * kPBytes);
#pragma unroll
              for (int mt = 0; mt < 4; ++mt)     // latent columns [128 mt, +128): c^KV chunks 2 mt, 2 mt + 1
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)   // tokens [16 kk, +16)
                  mma_ss(tmem + kTmemO + mt * kNH, sdesc_sw128(st + 2 * mt * kChunk + kk * 2048, kChunk, 1024),
                         sdesc_sw128(pb + kk * 32, 16, 1024), idesc_pv, (npv > 0 || kk > 0) ? 1u : 0u);
              mma_commit(&p_free[b]);
              mma_commit(&empty[s]);
              if (npv == nt - 1) mma_commit(o_done);
              ++npv;
              issued = true;
            }
          }
          if (!issued && ns < nt) {  // S^T(g) = C Q^T
            const int g = it + ns;
            const int s = g % kStages, b = g & 1;
            if (mbar_test_wait(smem_u32(&full[s]), (g / kStages) & 1) &&
                mbar_test_wait(smem_u32(&s_free[b]), ((g >> 1) & 1) ^ 1)) {
              tc_fence_after();
              const uint32_t st = smem_u32(stages + s * kStageBytes);
              for (int c = 0; c < 9; ++c) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_ss(tmem + kTmemS + b * kNH, sdesc_sw128(st + c * kChunk + kk * 32, 16, 1024),
                         sdesc_sw128(qb + c * kQChunk + kk * 32, 16, 1024), idesc_s, (c | kk) ? 1u : 0u);
              }
              mma_commit(&s_full[b]);
              if (ns == nt - 1) mma_commit(&q_free[piece & 1]);  // no MMA of this piece reads its Q any more
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
  } else {
    // ------------------------------------------------------------ Q, softmax, epilogue
    const int q4 = warp & 3;                  // TMEM lane quarter = tokens 16 q4 .. +15 of a tile
    const int tl16 = lane & 15, hg = lane >> 4;  // token within the quarter, head group (heads 8 hg .. +7)
    const uint32_t tq = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int tid = threadIdx.x - 64;         // 0 .. 127
    // Q of sequence b into buffer j: the B-operand chunks (16 heads x 576
    // columns, 128B swizzle), heads past n_h zero
    auto load_q = [&](int b, int j) {
      const __nv_bfloat16* qb = a.qlat + static_cast<long long>(b) * a.n_h * kRow;
      uint4 v[kNH * 72 / 128];
#pragma unroll
      for (int r = 0; r < kNH * 72 / 128; ++r) {  // 72 pieces of 16 bytes per head row
        const int i = tid + 128 * r, h = i / 72, pc = i % 72;
        v[r] = h < a.n_h ? *reinterpret_cast<const uint4*>(qb + h * kRow + pc * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int r = 0; r < kNH * 72 / 128; ++r) {
        const int i = tid + 128 * r, h = i / 72, pc = i % 72, c = pc >> 3, u = pc & 7;
        st_shared_v4(smem_u32(qs + j * kQBytes) + c * kQChunk + h * 128 + ((u ^ (h & 7)) << 4), v[r]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_full[j]);
    };
    static_assert(kNH * 72 % 128 == 0, "Q pieces per thread");
    // the worker's last tile: pieces after the current one are the next
    // sequences while their tiles start before it
    long long r1 = 0;
    {
      const long long T = a.tile_start[a.B];
      const int We = static_cast<int>(T < a.W ? T : a.W);
      if (T > 0 && w < We) r1 = worker_begin(w + 1, T, We);
    }
    int it = 0, piece = 0;
    for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
      if (*abort_flag) return;
      if (piece == 0) load_q(p.b, 0);  // later pieces' Q is loaded ahead, below
      const int L1 = a.seqlen[p.b] + 1;
      float m[8], l[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        m[j] = -INFINITY;
        l[j] = 0.f;
      }
      const int nt = p.t1 - p.t0;
      for (int k = 0; k < nt; ++k) {
        const int g = it + k, b = g & 1;
        const uint32_t ph = (g >> 1) & 1;
        if (!mbar_wait(&s_full[b], ph, wc)) return;
        tc_fence_after();
        uint32_t sr[8];
        tmem_ld16x2_x8(tq + kTmemS + b * kNH, sr);  // token 16 q4 + tl16, heads 8 hg .. +7
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[b]);
        const int tile0 = (p.t0 + k) * kTile;
        const int tok = 16 * q4 + tl16;           // token of the tile
        const bool valid = tile0 + tok < L1;
        float sc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) sc[j] = valid ? __uint_as_float(sr[j]) : -INFINITY;
        if (k == 0) {
          // the piece's reference: each head's max over the first tile's 64
          // tokens (16 lanes of each half warp, then the four warps)
          float mw[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float v = sc[j];
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            mw[j] = v;
          }
          float* mb = mxs + (piece & 1) * 4 * kNH;
          if (tl16 == 0)
#pragma unroll
            for (int j = 0; j < 8; ++j) mb[q4 * kNH + 8 * hg + j] = mw[j];
          __syncwarp();
          if (lane == 0) mbar_arrive(&mx_bar[piece & 1]);
          if (!mbar_wait(&mx_bar[piece & 1], (piece >> 1) & 1, wc)) return;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            m[j] = fmaxf(fmaxf(mb[8 * hg + j], mb[kNH + 8 * hg + j]), fmaxf(mb[2 * kNH + 8 * hg + j], mb[3 * kNH + 8 * hg + j]));
        }
        // P against the piece's reference, capped at 2^96 (a jump past it is reported)
        bool over = false;
#pragma unroll
        for (int j = 0; j < 8; ++j) over |= sc[j] > m[j] + kRangeLog2;
        if (__any_sync(0xffffffffu, over)) {
          if (over) atomicOr(a.status, FAULT_RANGE);
#pragma unroll
          for (int j = 0; j < 8; ++j) sc[j] = fminf(sc[j], m[j] + kRangeLog2);
        }
        float pv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          pv[j] = ex2_approx(sc[j] - m[j]);
          l[j] += pv[j];
        }
        const int v64 = min(kTile, L1 - tile0);  // valid rows of the tile
        // ---- P^T buffer b is free once PV(g - 2) retired
        if (!mbar_wait(&p_free[b], ph ^ 1, wc)) return;
        tc_fence_after();
        if (v64 < kTile) {
          // rows past the sequence may hold anything (even NaN); 0 * NaN would
          // poison O, so the c^KV rows the PV product reads are zeroed (the
          // tile's S products have retired: s_full)
          uint8_t* st = stages + (g % kStages) * kStageBytes;
          const int n16 = (kTile - v64) * 64;  // 16-byte pieces: 8 chunks x 8 per row
          for (int idx = tid; idx < n16; idx += 128) {
            const int row = v64 + (idx >> 6), c16 = idx & 63;
            *reinterpret_cast<uint4*>(st + (c16 >> 3) * kChunk + row * 128 + (c16 & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        // ---- P^T: head rows, token columns (128B swizzle); this thread's
        // token tok, heads 8 hg .. +7
        uint8_t* pt = pbuf + b * kPBytes;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int h = 8 * hg + j;
          reinterpret_cast<__nv_bfloat16*>(pt + h * 128 + (((tok >> 3) ^ (h & 7)) << 4))[tok & 7] =
              __float2bfloat16_rn(pv[j]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
      }
      // ---- the next piece's Q into the other buffer, so that its S products
      // run during this piece's epilogue (the buffer's piece - 1 S retired)
      if (p.b + 1 < a.B && a.tile_start[p.b + 1] < r1) {
        if (piece > 0 && !mbar_wait(&q_free[(piece + 1) & 1], ((piece - 1) >> 1) & 1, wc)) return;
        load_q(p.b + 1, (piece + 1) & 1);
      }
      // ---- epilogue of the piece: (m, l) per head to ml_part while the last
      // PV product runs, then O^T (latent rows in TMEM lanes) to o_part.
      // l per head: over the 16 tokens of each half warp, then the four warps
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = l[j];
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        l[j] = v;
      }
      if (tl16 == 0)
#pragma unroll
        for (int j = 0; j < 8; ++j) lxs[q4 * kNH + 8 * hg + j] = l[j];
      __syncwarp();
      if (lane == 0) mbar_arrive(l_bar);
      if (!mbar_wait(l_bar, piece & 1, wc)) return;
      if (warp == 2 && lane < kNH && lane < a.n_h) {
        const float* mb = mxs + (piece & 1) * 4 * kNH;
        const float mh = fmaxf(fmaxf(mb[lane], mb[kNH + lane]), fmaxf(mb[2 * kNH + lane], mb[3 * kNH + lane]));
        const float lh = ((lxs[lane] + lxs[kNH + lane]) + lxs[2 * kNH + lane]) + lxs[3 * kNH + lane];
        a.ml_part[(static_cast<long long>(p.slot) * a.n_h + lane) * 2] = mh;
        a.ml_part[(static_cast<long long>(p.slot) * a.n_h + lane) * 2 + 1] = lh;
      }
      if (!mbar_wait(o_done, piece & 1, wc)) return;
      tc_fence_after();
      {
        float o[4][16];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) tmem_ld16(tq + kTmemO + mt * kNH, o[mt]);  // latent 128 mt + 32 q4 + lane
        tmem_wait_ld();
        float* op = a.o_part + static_cast<long long>(p.slot) * a.n_h * 512 + 32 * q4 + lane;
#pragma unroll
        for (int h = 0; h < kNH; ++h)
          if (h < a.n_h)
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) op[h * 512 + 128 * mt] = o[mt][h];
      }
      tc_fence_before();
      it += nt;
      ++piece;
    });
  }
  // ---- teardown: every MMA retired before TMEM is freed (bounded)
  if (threadIdx.x == 0) griddep_launch_dependents();
  if (warp == 1) {
    __syncwarp();
    if (lane == 0) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(smem_u32(drain), 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  }
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mla
