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
// tile feeds M = 128 MMAs instead of being read once per head.  The fp32
// latent accumulator O (128 heads x 512) fills a whole SM's tensor memory, so
// each worker is a cluster of two CTAs, and CTA r accumulates the columns
// O[:, 256r, 256r + 256).  The pair splits every 64-token tile by tokens for
// the scores: CTA r computes S for the tile's rows [32r, 32r + 32) over all
// 576 columns (tcgen05.mma, M = 128 heads, N = 32, K = 576), the two CTAs
// swap their per-head maxima of a piece's first tile (512 bytes) so both take
// the same reference, and each sends the bf16 P of its 32 rows (8 KB) into
// the partner's P buffer.
// Both then run O_r += P C_r over all 64 rows (N = 256): CTA r TMA-loads its
// own 32 rows whole and the partner's 32 rows in its own 256 columns, so the
// pair reads the partner-row columns twice, the second time from L2.  A PV
// retirement is committed to both CTAs' barriers (multicast commit), which
// tells each side that both P buffers may take the next tile.
//
// The softmax waits for the partner once per piece.  The max over both
// halves of a piece's first tile is the piece's reference m, and every P of
// the piece is 2^(s - m).  The reference cancels in O / l, so it need not be
// the running max: later tiles may give P > 1, and O and l are never
// rescaled.  The kernel's range is P <= 2^96 (ample for fp32 O and l); a
// tile whose scores rise past it sets FAULT_RANGE.
//
// Warp roles (448 threads per CTA; 704 for E4M3 rows):
//   warp 0      TMA producer (bf16 rows: the three rings below; E4M3 rows:
//               raw stages and bf16 stages)
//   warp 1      TMEM owner and MMA issuer: S(j) once tile j landed and the S
//               buffer was read out, PV(j) once both halves of P(j) are in place
//   warps 2-5   Q_lat of each piece: chunks 0-6 (bf16 pairs) into TMEM, chunks
//               7-8 into shared memory, both MMA A operands; for E4M3 rows
//               also a third of the decode of each raw stage into a bf16 stage
//   warps 6-13  softmax: warp 6+i and warp 10+i share lane quarter i mod 4,
//               16 heads each; two threads per head (rows 0-15 and 16-31 of
//               this CTA's half, via the 16-lane TMEM access shape).  Softmax
//               against the piece's reference max (above), and the per-piece
//               epilogue; CTA 1 sends its share of l to CTA 0.
//   warps 14-21 E4M3 rows only: the other two thirds of the decode
#pragma once
#include "mla.h"
#include "ptx.cuh"
#include "simt.cuh"

namespace mla {

constexpr int kAttnTileTokens = 64;
constexpr bool kAttnTcReady = true;

namespace attn {
constexpr int kHalf = 32;                              // rows of a tile whose scores one CTA computes
constexpr int kChunkBytes = kHalf * 128;               // 32 token rows x 64 latent columns, bf16, 128B swizzle
constexpr int kPeerChunks = 4;                         // partner's rows: this CTA's 256 c^KV columns
constexpr int kQTmemChunks = 7;                        // Q chunks held in TMEM; the rest in shared memory
constexpr int kQSmemChunks = 9 - kQTmemChunks;
constexpr int kQChunkBytes = 128 * 128;                // 128 heads x 64 columns, bf16
constexpr int kPBytes = 128 * 128;                     // P: 128 heads x 64 rows, bf16 (CTA 0's rows first)
constexpr int kMaxSlots = 4;                           // partner tile maxima in flight (tile j in slot j % 4)
constexpr int kAuxBytes = 3072;                        // partner maxima, CTA 1's l, barriers
// TMEM columns: O half [0,256), S [256,288), Q chunks 0-6 (bf16 pairs) [288,512)
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemQ = 288, kTmemCols = 512;
constexpr float kRangeLog2 = 96.f;                     // largest exponent of P before the max catches up
constexpr int kRow = 576;                              // d_c + d_R
static_assert(kTmemQ + kQTmemChunks * 32 == kTmemCols, "TMEM budget");

// Stage layouts of the two cache formats.  The MMAs always read bf16 tiles:
// the own rows' c^KV chunks 0-7 and k^R chunk 8, and the partner rows'
// chunks in this CTA's c^KV columns.  For bf16 rows the TMA loads them into
// three rings, each released as soon as its last reader retired (ring A: the
// own rows' chunks only the scores read; ring B: the own rows in this CTA's
// columns; ring C: the partner rows), which keeps more tiles in flight than
// whole 53 KB stages would in the same shared memory.  For E4M3 rows the TMA
// fills a raw stage (k^R chunk in bf16 with the 128B swizzle, the own rows'
// 512 code bytes as two boxes of 256, the partner rows' 256 code bytes in
// this CTA's columns, and the scale bytes of both), and the converter warps
// decode it into the bf16 stage; the S MMAs take k^R from the raw stage.
template <bool kFp8>
struct Cfg {
  static constexpr int kStages = kFp8 ? 2 : 3;           // bf16 stages
  static constexpr int kOwnChunks = kFp8 ? 8 : 9;        // own-row chunks in a bf16 stage
  static constexpr int kStageBytes = (kOwnChunks + kPeerChunks) * kChunkBytes;
  static constexpr int kRawStages = kFp8 ? 2 : 0;
  // raw stage: k^R chunk | own codes 0-255 | own codes 256-511 | partner codes | own scales | partner scales
  static constexpr int kRawKr = 0, kRawOwn0 = 4096, kRawOwn1 = 4096 + 8192, kRawPeer = 4096 + 2 * 8192;
  static constexpr int kRawOwnS = 4096 + 3 * 8192, kRawPeerS = kRawOwnS + 512;
  static constexpr int kRawTx = kRawPeerS + 512;         // bytes the TMA brings per raw stage
  static constexpr int kRawBytes = kFp8 ? 30720 : 0;     // rounded up to 1 KB (the swizzled chunk's alignment)
  // bf16 rows: three rings instead of whole stages, so that each part of a
  // tile is held only as long as it is read.  Ring A: the own rows' chunks
  // that only the scores read (the partner's c^KV columns and k^R), free
  // once S retires.  Ring B: the own rows in this CTA's columns (S and PV).
  // Ring C: the partner's rows in this CTA's columns (PV only), loaded when
  // the PV before frees its slot.
  static constexpr int kRingA = 2, kRingB = 5, kRingC = 2;
  static constexpr int kABytes = 5 * kChunkBytes, kBBytes = 4 * kChunkBytes, kCBytes = 4 * kChunkBytes;
  static constexpr int kStageRegion =
      kFp8 ? kStages * kStageBytes : kRingA * kABytes + kRingB * kBBytes + kRingC * kCBytes;
  static constexpr int kBars = kFp8 ? kStages : kRingA + kRingB + kRingC;  // full / empty barriers of the rings
  static_assert(kFp8 || (kRingB >= kRingC && kRingB - kRingC < 8), "ring C trails ring B by fewer than 8 tiles");
  // Ring C's load of tile g is issued with ring B's load of tile g + kRingB -
  // kRingC, after ring A's load of tile g + kRingB - kRingC - 1, which waits
  // for S(g + kRingB - kRingC - 1 - kRingA).  The last tile g of a piece needs
  // its ring C load before the next piece's first S can issue, so that S
  // index must not pass g.
  static_assert(kFp8 || kRingB <= kRingA + kRingC + 1, "ring C's loads must not wait for a later piece");
  // P buffers: P(g) is written once PV(g - kPBufs) retired in both CTAs
  static constexpr int kPBufs = 2;
  // E4M3 rows: the decode, bound by its latency rather than its arithmetic,
  // is split over twelve warps, the four Q warps and eight more (warps
  // 14-21) that do nothing else
  static constexpr int kConvWarps = kFp8 ? 12 : 0;
  static constexpr int kThreads = kFp8 ? 704 : 448;
  // stages (rings) | raw stages | Q chunks 7-8 | P x 2 | aux
  static constexpr int kSmem = 1024 + kStageRegion + kRawStages * kRawBytes + kQSmemChunks * kQChunkBytes +
                               kPBufs * kPBytes + kAuxBytes;
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(!kFp8 || kRawTx <= kRawBytes, "raw stage");
};
}  // namespace attn

struct AttnArgs {
  CUtensorMap map_cache;       // bf16 view of the rows, box {64 columns, 32 rows}, 128B swizzle (E4M3 rows: k^R only)
  CUtensorMap map_code;        // E4M3 rows: bytes, box {256, 32}, no swizzle
  CUtensorMap map_scale;       // E4M3 rows: bytes, box {16, 32} at the scale byte, no swizzle
  int kr_x;                    // E4M3 rows: k^R's column in the bf16 view (d_c / 2)
  int scale_x;                 // E4M3 rows: byte of the scale exponent
  const __nv_bfloat16* qlat;   // [B][n_h][576]
  CacheLayout lay;             // cache rows of each sequence (contiguous or paged)
  long long n_rows;            // rows of the cache tensor
  const int32_t* seqlen;
  const int* tile_start;
  const int* seg_start;
  int B, W, n_h;
  float* o_part;               // [slots][n_h][512]
  float* ml_part;              // [slots][n_h][2]
  int* status;
};

// Decodes 8 E4M3 codes scaled by 2^k into 8 bf16 (exact: a code value times
// a power of two fits bf16's 8-bit significand).
__device__ __forceinline__ uint4 e4m3x8_to_bf16(uint2 raw, float scale) {
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t word = i < 2 ? raw.x : raw.y;
    const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>((word >> (16 * (i & 1))) & 0xFFFFu);
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * scale, f.y * scale);
    out[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(attn::Cfg<kFp8>::kThreads, 1)
    attn_decode_tc_kernel(const __grid_constant__ AttnArgs a) {
  using namespace attn;
  using C = Cfg<kFp8>;
  constexpr int kStages = C::kStages;
  constexpr int kOwnChunks = C::kOwnChunks;
  constexpr int kStageBytes = C::kStageBytes;
  constexpr int kRS = C::kRawStages > 0 ? C::kRawStages : 1;  // raw-stage modulus (unused for bf16 rows)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* stages = smem;
  uint8_t* raws = stages + C::kStageRegion;          // E4M3 rows: raw stages (TMA)
  uint8_t* qs = raws + C::kRawStages * C::kRawBytes;  // Q chunks 7-8, MMA A operand
  uint8_t* pbuf = qs + kQSmemChunks * kQChunkBytes;   // [kPBufs] P (bf16), MMA A operand
  uint8_t* aux = pbuf + C::kPBufs * kPBytes;
  float* mx = reinterpret_cast<float*>(aux);          // [4][128] the partner's tile maxima (st.async)
  float* lsh = mx + kMaxSlots * 128;                  // [128] CTA 1's share of l, in CTA 0 (st.async)
  uint64_t* full = reinterpret_cast<uint64_t*>(aux + 2560);
  uint64_t* empty = full + C::kBars;
  uint64_t* s_full = empty + C::kBars;  // S(j) in TMEM (MMA -> softmax)
  uint64_t* s_free = s_full + 1;       // S read out (softmax -> MMA)
  uint64_t* mx_full = s_free + 1;      // [4] the partner's maxima of tile j landed (slot j % 4)
  constexpr int kPB = C::kPBufs;
  uint64_t* p_full = mx_full + kMaxSlots;  // [kPB] this CTA's half of P(j) written (buffer j % kPB)
  uint64_t* px_full = p_full + kPB;    // [kPB] the partner's half of P(j) landed
  uint64_t* pv_done = px_full + kPB;   // [kPB] PV(j) retired in both CTAs (one commit from each)
  uint64_t* q_full = pv_done + kPB;
  uint64_t* q_free = q_full + 1;       // last S of the piece retired (MMA -> Q warps)
  uint64_t* o_done = q_free + 1;
  uint64_t* l_full = o_done + 1;       // CTA 0: CTA 1's l of the piece landed
  uint64_t* drain = l_full + 1;
  uint64_t* raw_full = drain + 1;      // [2] E4M3 rows: raw stage loaded (TMA)
  uint64_t* raw_empty = raw_full + 2;  // [2] E4M3 rows: raw stage read by the converter and by S's k^R MMAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(raw_empty + 2);
  static_assert(2560 + (2 * C::kBars + 15 + 3 * C::kPBufs) * 8 + 8 <= kAuxBytes, "aux layout: maxima, l, barriers");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int w = blockIdx.x >> 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kBars; ++s) {
      mbar_init(&full[s], kFp8 ? C::kConvWarps : 1);  // E4M3 rows: one arrival per converter warp
      mbar_init(&empty[s], 1);
    }
    for (int r = 0; r < C::kRawStages; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], C::kConvWarps + 1);  // the converter warps and the commit after S
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);        // one arrival per softmax warp
    for (int i = 0; i < kMaxSlots; ++i) mbar_init(&mx_full[i], 1);  // armed per phase with the partner's 512 bytes
    for (int i = 0; i < kPB; ++i) {
      mbar_init(&p_full[i], 8);   // one arrival per softmax warp
      mbar_init(&px_full[i], 1);  // armed per phase with the partner's 8 KB
      mbar_init(&pv_done[i], 2);  // this CTA's and the partner's PV commit
    }
    mbar_init(q_full, 128);
    mbar_init(q_free, 1);
    mbar_init(o_done, 1);
    mbar_init(l_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (int i = 0; i < kMaxSlots; ++i) mbar_arrive_expect_tx(&mx_full[i], 128 * 4);
    for (int i = 0; i < kPB; ++i) mbar_arrive_expect_tx(&px_full[i], kPBytes / 2);
    if (rank == 0) mbar_arrive_expect_tx(l_full, 128 * 4);
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&a.map_cache);
    if (kFp8) {
      prefetch_tmap(&a.map_code);
      prefetch_tmap(&a.map_scale);
    }
  }
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
  // bf16 rows: slots of tile g in the three rings, and their barriers
  constexpr int kRA = C::kRingA, kRB = C::kRingB, kRC = C::kRingC;
  uint8_t* const ring_a = stages;
  uint8_t* const ring_b = ring_a + kRA * C::kABytes;
  uint8_t* const ring_c = ring_b + kRB * C::kBBytes;
  auto slot_a = [&](int g) { return ring_a + (g % kRA) * C::kABytes; };
  auto slot_b = [&](int g) { return ring_b + (g % kRB) * C::kBBytes; };
  auto slot_c = [&](int g) { return ring_c + (g % kRC) * C::kCBytes; };
  auto bar_a = [&](int g) { return g % kRA; };
  auto bar_b = [&](int g) { return kRA + g % kRB; };
  auto bar_c = [&](int g) { return kRA + kRB + g % kRC; };

  // E4M3 rows: decode raw stage cv into its bf16 stage, warp cw's share.  A
  // task is 512 codes: one own row (lanes 0-15 its codes 0-255, lanes 16-31
  // its codes 256-511) or two partner rows (one per half warp); a lane reads
  // 16 codes (16 contiguous bytes) and writes two 16-byte pieces of one
  // swizzled chunk row.  Warp cw takes tasks cw + kConvWarps i; their code
  // and scale loads are all issued before any conversion.
  auto convert_tile = [&](int cw, int cv) -> bool {
    constexpr int kCW = C::kConvWarps > 0 ? C::kConvWarps : 1;
    constexpr int kTasks = kHalf + kHalf / 2, kBatch = kTasks / kCW;
    static_assert(!kFp8 || kTasks == kCW * kBatch, "converter tasks");
    const int hl = lane >> 4, l16 = lane & 15;
    const int r = cv % kRS, s = cv % kStages;
    if (!mbar_wait(&raw_full[r], (cv / kRS) & 1, wc)) return false;
    if (!mbar_wait(&empty[s], ((cv / kStages) & 1) ^ 1, wc)) return false;
    const uint8_t* raw = raws + r * C::kRawBytes;
    uint8_t* st = stages + s * kStageBytes;
    uint4 codes[kBatch];
    float scl[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int task = cw + kCW * i;
      const bool own = task < kHalf;
      const int row = own ? task : 2 * (task - kHalf) + hl;
      const uint8_t* src = raw + (own ? (hl ? C::kRawOwn1 : C::kRawOwn0) : C::kRawPeer) + row * 256 + l16 * 16;
      codes[i] = *reinterpret_cast<const uint4*>(src);
      const int k = static_cast<int8_t>(raw[(own ? C::kRawOwnS : C::kRawPeerS) + row * 16]);
      scl[i] = k >= -126 ? __int_as_float((k + 127) << 23) : ldexpf(1.f, k);  // 2^k
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int task = cw + kCW * i;
      const bool own = task < kHalf;
      const int row = own ? task : 2 * (task - kHalf) + hl;
      const uint4 lo = e4m3x8_to_bf16(make_uint2(codes[i].x, codes[i].y), scl[i]);
      const uint4 hi = e4m3x8_to_bf16(make_uint2(codes[i].z, codes[i].w), scl[i]);
      // columns 16 l16 .. +15 of the 256-column segment: chunk l16 / 4,
      // pieces 2 (l16 % 4) and +1; the half warps store opposite parities
      // first, so each store spreads over all banks
      const int chunk = (own ? 4 * hl : kOwnChunks) + (l16 >> 2);
      uint8_t* dst = st + chunk * kChunkBytes + row * 128;
      const int pc = 2 * (l16 & 3), sw = row & 7, f = hl ^ (row & 1);
      *reinterpret_cast<uint4*>(dst + (((pc + f) ^ sw) << 4)) = f ? hi : lo;
      *reinterpret_cast<uint4*>(dst + (((pc + (f ^ 1)) ^ sw) << 4)) = f ? lo : hi;
    }
    fence_proxy_async_smem();  // the MMAs read the stage through the async proxy
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&full[s]);
      mbar_arrive(&raw_empty[r]);
    }
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      // Bytes the partner also loads keep the normal L2 priority, so that the
      // second read is an L2 hit; the rest is streamed with evict-first.
      const uint64_t pol_once = policy_evict_first();
      const uint64_t pol_twice = policy_evict_normal();
      int it = 0;
      int n_a = 0, n_b = 0, n_c = 0;  // bf16 rows: loads issued into each ring
      int yp_hist[8];                 // bf16 rows: the partner rows' start of the last 8 tiles
      // bf16 rows: ring C's chunks of tile gc (the partner's rows in this CTA's columns)
      auto load_c = [&](int gc) -> bool {
        if (!mbar_wait(&empty[bar_c(gc)], ((gc / kRC) & 1) ^ 1, wc)) return false;
        mbar_arrive_expect_tx(&full[bar_c(gc)], C::kCBytes);
        for (int j = 0; j < 4; ++j)
          tma_load_2d(slot_c(gc) + j * kChunkBytes, &a.map_cache, &full[bar_c(gc)],
                      (4 * static_cast<int>(rank) + j) * 64, yp_hist[gc & 7], pol_twice);
        ++n_c;
        return true;
      };
      for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
        if (*abort_flag) return;
        const long long row0 = a.lay.block_table ? 0 : a.lay.seq_start[p.b];  // contiguous layout
        for (int t = p.t0; t < p.t1; ++t, ++it) {
          // a tile lies within one page; a tile without a page (a capacity
          // fault of the call) loads rows past the tensor, which read as zero
          long long y0 = a.lay.block_table ? a.lay.row(p.b, static_cast<long long>(t) * kAttnTileTokens)
                                           : row0 + static_cast<long long>(t) * kAttnTileTokens;
          if (y0 < 0) y0 = a.n_rows;
          if constexpr (kFp8) {
            const int r = it % kRS;
            if (!mbar_wait(&raw_empty[r], ((it / kRS) & 1) ^ 1, wc)) return;
            mbar_arrive_expect_tx(&raw_full[r], C::kRawTx);
            uint8_t* dst = raws + r * C::kRawBytes;
            const int y_own = static_cast<int>(y0 + kHalf * rank), y_peer = static_cast<int>(y0 + kHalf * peer);
            tma_load_2d(dst + C::kRawKr, &a.map_cache, &raw_full[r], a.kr_x, y_own, pol_once);
            // the partner reads this CTA's rows in its own half of the codes too
            tma_load_2d(dst + C::kRawOwn0, &a.map_code, &raw_full[r], 0, y_own, peer == 0 ? pol_twice : pol_once);
            tma_load_2d(dst + C::kRawOwn1, &a.map_code, &raw_full[r], 256, y_own, peer == 1 ? pol_twice : pol_once);
            tma_load_2d(dst + C::kRawPeer, &a.map_code, &raw_full[r], 256 * static_cast<int>(rank), y_peer, pol_twice);
            tma_load_2d(dst + C::kRawOwnS, &a.map_scale, &raw_full[r], a.scale_x, y_own, pol_twice);
            tma_load_2d(dst + C::kRawPeerS, &a.map_scale, &raw_full[r], a.scale_x, y_peer, pol_twice);
            continue;
          }
          // tile it: ring C's chunks of tile it - (kRB - kRC) first (its slot
          // frees with the same PV as ring B's slot of tile it), then ring A
          // (the own rows' score-only chunks) and ring B (the own rows in this
          // CTA's columns)
          const int y_own = static_cast<int>(y0 + kHalf * rank), y_peer = static_cast<int>(y0 + kHalf * peer);
          yp_hist[it & 7] = y_peer;
          if (it - (kRB - kRC) >= 0 && !load_c(it - (kRB - kRC))) return;
          if (!mbar_wait(&empty[bar_a(it)], ((it / kRA) & 1) ^ 1, wc)) return;
          mbar_arrive_expect_tx(&full[bar_a(it)], C::kABytes);
          for (int j = 0; j < 4; ++j)  // the partner reads these rows in its columns too
            tma_load_2d(slot_a(it) + j * kChunkBytes, &a.map_cache, &full[bar_a(it)], (4 * static_cast<int>(peer) + j) * 64,
                        y_own, pol_twice);
          tma_load_2d(slot_a(it) + 4 * kChunkBytes, &a.map_cache, &full[bar_a(it)], 512, y_own, pol_once);
          ++n_a;
          if (!mbar_wait(&empty[bar_b(it)], ((it / kRB) & 1) ^ 1, wc)) return;
          mbar_arrive_expect_tx(&full[bar_b(it)], C::kBBytes);
          for (int j = 0; j < 4; ++j)
            tma_load_2d(slot_b(it) + j * kChunkBytes, &a.map_cache, &full[bar_b(it)], (4 * static_cast<int>(rank) + j) * 64,
                        y_own, pol_once);
          ++n_b;
        }
      });
      if constexpr (!kFp8) {
        for (int gc = it - (kRB - kRC) > 0 ? it - (kRB - kRC) : 0; gc < it && !*abort_flag; ++gc)
          if (!load_c(gc)) break;
      }
      // every load issued has landed before the CTA may leave (after an abort,
      // loads can still be in flight into stages nobody consumes)
      if constexpr (kFp8) {
        drain_ring(raw_full, kRS, it);
      } else {
        drain_ring(full + bar_a(0), kRA, n_a);
        drain_ring(full + bar_b(0), kRB, n_b);
        drain_ring(full + bar_c(0), kRC, n_c);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_bf16(128, kHalf, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 256, false, true);
      int it = 0, piece = 0;
      for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
        if (*abort_flag) return;
        if (!mbar_wait(q_full, piece & 1, wc)) return;
        tc_fence_after();
        const int nt = p.t1 - p.t0;
        int ns = 0, npv = 0;
        uint32_t spins = 0;
        uint64_t t_idle = 0;
        while (npv < nt) {
          bool issued = false;
          if (npv < ns) {
            const int g = it + npv;
            const int s = g % kStages;
            const int b = g % kPB;
            const uint32_t ph = (g / kPB) & 1;
            // bf16 rows: the partner rows' chunks come with ring C
            const bool c_ready = kFp8 || mbar_test_wait(smem_u32(&full[bar_c(g)]), (g / kRC) & 1);
            if (c_ready && mbar_test_wait(smem_u32(&p_full[b]), ph) &&
                mbar_test_wait_cluster(smem_u32(&px_full[b]), ph)) {
              tc_fence_after();
              fence_proxy_async_smem();  // the partner's half came in through st.async
              // next phase: the partner's half of P(g + kPB), which it sends
              // only after this PV retired
              mbar_arrive_expect_tx(&px_full[b], kPBytes / 2);
              const uint32_t st = smem_u32(stages + s * kStageBytes);
              // own rows and partner rows, this CTA's c^KV columns
              const uint32_t own_rows = kFp8 ? st + 4 * rank * kChunkBytes : smem_u32(slot_b(g));
              const uint32_t peer_rows = kFp8 ? st + kOwnChunks * kChunkBytes : smem_u32(slot_c(g));
              const uint32_t pb = smem_u32(pbuf + b * kPBytes);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {  // rows [16 kk, 16 kk + 16) of the tile; CTA 0's rows first
                const uint32_t rows = (kk >> 1) == static_cast<int>(rank) ? own_rows : peer_rows;
                mma_ss(tmem + kTmemO, sdesc_sw128(pb + kk * 32, 16, 1024),
                       sdesc_sw128(rows + (kk & 1) * 2048, kChunkBytes, 1024), idesc_pv, (npv > 0 || kk > 0) ? 1u : 0u);
              }
              mma_commit_multicast(&pv_done[b], 0x3);  // P buffer b is free in both CTAs once both commits land
              if constexpr (kFp8) {
                mma_commit(&empty[s]);
              } else {
                mma_commit(&empty[bar_b(g)]);
                mma_commit(&empty[bar_c(g)]);
              }
              if (npv == nt - 1) mma_commit(o_done);
              ++npv;
              issued = true;
            }
          }
          if (!issued && ns < nt) {
            const int g = it + ns;
            const int s = g % kStages;
            const bool data = kFp8 ? mbar_test_wait(smem_u32(&full[s]), (g / kStages) & 1)
                                   : mbar_test_wait(smem_u32(&full[bar_a(g)]), (g / kRA) & 1) &&
                                         mbar_test_wait(smem_u32(&full[bar_b(g)]), (g / kRB) & 1);
            if (data && mbar_test_wait(smem_u32(s_free), (g & 1) ^ 1)) {
              tc_fence_after();
              const uint32_t st = smem_u32(stages + s * kStageBytes);
              // the own rows' chunk ci (64 columns; 8 = k^R): E4M3 rows keep
              // c^KV in the bf16 stage and k^R in the raw stage; bf16 rows
              // keep this CTA's columns in ring B and the rest in ring A
              auto own_chunk = [&](int ci) -> uint32_t {
                if constexpr (kFp8) {
                  return ci == 8 ? smem_u32(raws + (g % kRS) * C::kRawBytes + C::kRawKr) : st + ci * kChunkBytes;
                } else {
                  const int r4 = 4 * static_cast<int>(rank);
                  if (ci >= r4 && ci < r4 + 4) return smem_u32(slot_b(g)) + (ci - r4) * kChunkBytes;
                  return smem_u32(slot_a(g)) + (ci < 8 ? ci - 4 * static_cast<int>(peer) : 4) * kChunkBytes;
                }
              };
              const uint32_t dS = tmem + kTmemS;
              for (int ci = 0; ci < kQTmemChunks; ++ci) {
                const uint32_t bchunk = own_chunk(ci);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  mma_ts(dS, tmem + kTmemQ + ci * 32 + kk * 8, sdesc_sw128(bchunk + kk * 32, 16, 1024),
                         idesc_s, (ci | kk) ? 1u : 0u);
                }
              }
              for (int ci = 0; ci < kQSmemChunks; ++ci) {
                const uint32_t bchunk = own_chunk(kQTmemChunks + ci);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  mma_ss(dS, sdesc_sw128(smem_u32(qs) + ci * kQChunkBytes + kk * 32, 16, 1024),
                         sdesc_sw128(bchunk + kk * 32, 16, 1024), idesc_s, 1u);
                }
              }
              mma_commit(s_full);
              if constexpr (kFp8) mma_commit(&raw_empty[g % kRS]);  // the raw stage's k^R was read
              else mma_commit(&empty[bar_a(g)]);                     // ring A is read by S only
              if (ns == nt - 1) mma_commit(q_free);  // no MMA of this piece reads Q any more
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
    // ------------------------------------------------------------ Q_lat of each piece (and, for
    // E4M3 rows, the decode of every raw stage of the piece)
    const int q4 = warp & 3;
    const int h = q4 * 32 + lane;  // head = TMEM lane
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int sw = h & 7;
    const uint32_t q_row = smem_u32(qs) + h * 128;
    int piece = 0;
    int cv = 0;  // E4M3 rows: tiles converted so far
    for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
      if (*abort_flag) return;
      // the previous piece's S products have retired: nothing reads Q now
      if (piece > 0 && !mbar_wait(q_free, (piece - 1) & 1, wc)) return;
      tc_fence_after();
      const bool head = h < a.n_h;
      const __nv_bfloat16* qrow = a.qlat + (static_cast<long long>(p.b) * a.n_h + (head ? h : 0)) * kRow;
      for (int ci = 0; ci < kQTmemChunks; ++ci) {
        const uint4* src = reinterpret_cast<const uint4*>(qrow + ci * 64);
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = head ? src[i] : make_uint4(0, 0, 0, 0);
          r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
        }
        tmem_st32(tl + kTmemQ + ci * 32, r);
      }
      for (int ci = 0; ci < kQSmemChunks; ++ci) {  // 128-byte swizzled rows
        const uint4* src = reinterpret_cast<const uint4*>(qrow + (kQTmemChunks + ci) * 64);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          st_shared_v4(q_row + ci * kQChunkBytes + ((i ^ sw) << 4), head ? src[i] : make_uint4(0, 0, 0, 0));
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(q_full);
      ++piece;
      if constexpr (kFp8) {
        // ---- E4M3 rows: this warp's share of the decode of the piece's tiles
        for (int t = p.t0; t < p.t1; ++t, ++cv)
          if (!convert_tile(warp - 2, cv)) return;
      }
    });
  } else if (warp >= 14) {
    // ------------------------------------------------------------ E4M3 rows: the
    // other converter warps
    int cv = 0;
    for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
      if (*abort_flag) return;
      for (int t = p.t0; t < p.t1; ++t, ++cv)
        if (!convert_tile(4 + warp - 14, cv)) return;
    });
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp & 3;
    const int hs = (warp - 6) >> 2;  // which 16 heads of the lane quarter
    const int th = lane >> 4;        // rows [16 th, 16 th + 16) of this CTA's half
    const int h = q4 * 32 + hs * 16 + (lane & 15);
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32 + hs * 16) << 16);
    const int sw = h & 7;
    const bool lead = warp == 6 && lane == 0;  // re-arms the barriers the partner completes
    const uint32_t p_row = smem_u32(pbuf) + h * 128;
    const uint32_t p_row_peer = mapa(p_row, peer);
    const uint32_t pxfull_peer = mapa(smem_u32(px_full), peer);
    const uint32_t mx_peer = mapa(smem_u32(mx), peer) + h * 4;
    const uint32_t mxfull_peer = mapa(smem_u32(mx_full), peer);
    int it = 0, piece = 0;
    // The partner's maxima of the first tile of piece j sit in slot j % kMaxSlots.
    auto partner_max = [&](int j, float& v) -> bool {
      const int slot = j & (kMaxSlots - 1);
      if (!mbar_wait<true>(&mx_full[slot], (j / kMaxSlots) & 1, wc)) return false;
      v = mx[slot * 128 + h];
      // next phase of the slot: the partner's maxima of piece j + 4, which it
      // sends only after it received P of piece j + 1 from this CTA
      if (lead) mbar_arrive_expect_tx(&mx_full[slot], 128 * 4);
      return true;
    };
    for_each_piece(w, a.W, a.B, a.tile_start, a.seg_start, [&](const Piece& p) {
      if (*abort_flag) return;
      const bool head = h < a.n_h;
      const int L1 = a.seqlen[p.b] + 1;
      float m_run = -INFINITY, l_run = 0.f;  // l_run: this thread's 16 rows only
      const int nt = p.t1 - p.t0;
      for (int k = 0; k < nt; ++k) {
        const int g = it + k;
        const int b = g % kPB;
        const uint32_t ph = (g / kPB) & 1;
        if (!mbar_wait(s_full, g & 1, wc)) return;
        tc_fence_after();
        uint32_t sr[16];
        tmem_ld16x2(tl + kTmemS, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        const int tile0 = (p.t0 + k) * kAttnTileTokens;
        const int valid = min(16, L1 - (tile0 + kHalf * static_cast<int>(rank) + 16 * th));  // may be <= 0
        float sc[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) sc[j] = __uint_as_float(sr[j]);
        if (__any_sync(0xffffffffu, valid < 16)) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j >= valid) sc[j] = -INFINITY;
        }
        float mo = sc[0];
#pragma unroll
        for (int j = 1; j < 16; ++j) mo = fmaxf(mo, sc[j]);
        mo = fmaxf(mo, __shfl_xor_sync(0xffffffffu, mo, 16));  // this CTA's 32 rows
        if (k == 0) {
          // the piece's first tile sets its reference max: both halves of the
          // tile are needed, so the pair swaps its maxima once per piece
          if (th == 0)
            st_async_b32(mx_peer + (piece & (kMaxSlots - 1)) * 512, __float_as_uint(mo),
                         mxfull_peer + (piece & (kMaxSlots - 1)) * 8);
          float pm;
          if (!partner_max(piece, pm)) return;
          m_run = fmaxf(mo, pm);
        }
        // P of this thread's rows against the piece's reference max, and their
        // sum; exponents are capped at the kernel's range (a jump past it is
        // reported)
        if (__any_sync(0xffffffffu, mo > m_run + kRangeLog2)) {
          if (mo > m_run + kRangeLog2) atomicOr(a.status, FAULT_RANGE);
#pragma unroll
          for (int j = 0; j < 16; ++j) sc[j] = fminf(sc[j], m_run + kRangeLog2);
        }
        uint32_t pk[8];
        float lsum = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float p0 = ex2_approx(sc[2 * j] - m_run), p1 = ex2_approx(sc[2 * j + 1] - m_run);
          lsum += p0 + p1;
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          pk[j] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        l_run += lsum;
        // ---- P buffer b is free in both CTAs once PV(g - kPB) retired in both
        if (!mbar_wait_inline(&pv_done[b], ph ^ 1, wc)) return;
        tc_fence_after();
        const int v64 = min(kAttnTileTokens, L1 - tile0);  // valid rows of the tile
        if (v64 < kAttnTileTokens) {
          // rows past the sequence may hold anything (even NaN); 0 * NaN would
          // poison O, so the rows this CTA multiplies into O are zeroed
          uint8_t* st = stages + (g % kStages) * kStageBytes;
          // bf16 rows: the partner rows' chunks come with ring C, maybe later.
          // A parity wait only tells apart phases one apart, so the slot's
          // previous load (tile g - kRC) must have landed first: its PV has
          // retired (PV(g - kPB) did, above; a later one is waited for here).
          if constexpr (!kFp8) {
            if (kRC < kPB && g >= kRC &&
                !mbar_wait_inline(&pv_done[(g - kRC) % kPB], ((g - kRC) / kPB) & 1, wc))
              return;
            if (!mbar_wait(&full[bar_c(g)], (g / kRC) & 1, wc)) return;
          }
          const int n16 = (kAttnTileTokens - v64) * 32;  // 16-byte pieces: 4 chunks x 8 per row
          for (int idx = (warp - 6) * 32 + lane; idx < n16; idx += 256) {
            const int row = v64 + (idx >> 5), c16 = idx & 31;
            const bool own = (row >> 5) == static_cast<int>(rank);
            uint8_t* base = kFp8 ? st + (own ? 4 * static_cast<int>(rank) : kOwnChunks) * kChunkBytes
                                 : (own ? slot_b(g) : slot_c(g));
            *reinterpret_cast<uint4*>(base + (c16 >> 3) * kChunkBytes + (row & 31) * 128 + (c16 & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
        // ---- this CTA's half of P(g): rows [32 rank + 16 th, +16) of the tile,
        // into the local buffer and the partner's
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const uint32_t off = b * kPBytes + (((4 * rank + 2 * th + i) ^ sw) << 4);
          const uint4 v = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          st_async_v4(p_row_peer + off, v, pxfull_peer + b * 8);
          st_shared_v4(p_row + off, v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
      }
      // ---- epilogue of the piece: unnormalised O_r; CTA 0 writes m and l
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
      const float l_head = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);  // this CTA's 32 rows of each tile
      if (rank == 1) {
        if (th == 0) st_async_b32(mapa(smem_u32(lsh), peer) + h * 4, __float_as_uint(l_head), mapa(smem_u32(l_full), peer));
      } else {
        if (!mbar_wait<true>(l_full, piece & 1, wc)) return;
        if (th == 0 && head) {
          a.ml_part[(static_cast<long long>(p.slot) * a.n_h + h) * 2] = m_run;
          a.ml_part[(static_cast<long long>(p.slot) * a.n_h + h) * 2 + 1] = l_head + lsh[h];
        }
        // next phase: CTA 1's l of the next piece, which needs this CTA's P of
        // that piece first
        if (lead) mbar_arrive_expect_tx(l_full, 128 * 4);
      }
      tc_fence_before();
      it += nt;
      ++piece;
    });
    // The partner's PV commits for the last uses of the P buffers land in
    // this CTA's shared memory: they must have arrived before the CTA may exit.
    if (lead && !*abort_flag) {
      for (int b = 0; b < kPB; ++b) {
        const int uses = (it + kPB - 1 - b) / kPB;  // tiles g < it with g % kPB == b
        if (uses > 0 && !mbar_wait<true>(&pv_done[b], (uses - 1) & 1, wc)) break;
      }
    }
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
