// uv_combine.cuh -- the split-KV combine and the absorbed W_UV product of a
// decode step in one kernel ("DeepSeek-V2 summary" (7shi.hateblo.jp), App. C:
// the output o_t,i = W_UV_i sum_j softmax_j c^KV_j, with W_UV absorbed after
// the attention over the latents):
//
//   o_lat[b,i] = sum_s 2^(m_s - M) O_s[i]  /  sum_s 2^(m_s - M) l_s     (M = max_s m_s)
//   o[b,i]     = W_UV_i o_lat[b,i]
//
// over the pieces s of sequence b, from the attention kernel's unnormalised
// partials O_s (fp32) and (m_s, l_s).  One CTA per (head i, 64 sequences):
// sixteen warps combine the partials straight into the MMA's B operand in
// shared memory (64 tokens x 512 latent columns, bf16, 128B swizzle, one K
// block of 64 columns at a time so the MMAs start on the first block), while
// the TMA streams the head's 128 x 512 block of W_UV through a 3-slot ring
// (small enough that the next GEMM's CTAs fit beside this one's and fetch
// their weights early); one thread issues
// M = 128 (d_h rows), N = 64 tcgen05 MMAs over the 8 K blocks, and the
// epilogue writes o through the GEMM's per-head epilogue.  The normalised
// latents are also written out (bf16), as the separate combine did.
//
// The combine's arithmetic is the two-kernel path's: the same weights, the
// same accumulation order over the pieces, the same rounding to bf16.  Warp
// roles: warp 0 TMA, warp 1 TMEM owner and MMA issuer, warps 2 .. 17 combine,
// warps 2-5 then the epilogue.
//
// Few (head, 64-sequence) tiles (V2-Lite's 16 heads at B <= 64 make 16 CTAs
// on 148 SMs) split the 8 K blocks over a cluster of ks <= 4 CTAs along grid z:
// CTA z combines and multiplies K blocks [8 z / ks, 8 (z + 1) / ks) only,
// stages its fp32 partial tile in the idle W_UV ring, and after a cluster
// barrier sums rows [128 z / ks, 128 (z + 1) / ks) of the tile over the ks
// partials, in split order, through distributed shared memory before its
// epilogue on those rows.  At V2-Lite B = 32, four splits took a decode step
// from 84.0 to 79.5 us; eight (one K block per CTA) took it to 86.3 us, the
// cluster barriers and the reduction then costing more than the combine saves.
#pragma once
#include <type_traits>

#include "epilogue.cuh"

namespace mla {

struct UvCombineArgs {
  CUtensorMap mapA;      // W_UV [n_h d_h][d_c] bf16, box {64, 128}, 128B swizzle
  const float* o_part;   // [slots][n_h][512] unnormalised partial latent outputs
  const float* ml_part;  // [slots][n_h][2] (m, l) of each partial
  const int* seg_start;  // [N + 1] first slot of each sequence
  int n_h, N;            // heads, sequences (tokens)
  int ks;                // K splits per tile: the cluster size along grid z (1, 2 or 4)
  __nv_bfloat16* olat;   // [N][n_h][512] the normalised latent outputs
  Epi epi;               // EPI_PER_HEAD into o [N][n_h d_h]
  TokenMap tok;
  int* status;
};

namespace uvc {
constexpr int kCombWarps = 16;          // warps that combine (warps 2 .. 2 + kCombWarps - 1)
constexpr int kThreads = 64 + 32 * kCombWarps;
constexpr int kTPR = kCombWarps * 32 / 64;  // combine threads per token
constexpr int kCPT = 64 / kTPR;             // columns of a K block per thread
constexpr int kF4 = kCPT / 4;               // float4 loads of a K block per thread and piece
constexpr int kKbPass = 4;                  // K blocks per pass: kKbPass * kF4 loads of each piece in flight
static_assert(kCPT % 8 == 0 && 8 % kKbPass == 0, "combine thread mapping");
constexpr int kKb = 8;                  // d_c / 64 K blocks
constexpr int kSlabA = 128 * 128;       // 128 rows x 64 columns bf16
constexpr int kSlabB = 64 * 128;        // 64 tokens x 64 columns bf16
constexpr int kUnroll = 2;              // pieces whose loads are in flight together
constexpr int kRingA = 3;               // W_UV K blocks in flight
constexpr int kMaxKs = 4;               // K splits of a tile: two K blocks per CTA at most
constexpr int kSmem = 1024 + kRingA * kSlabA + kKb * kSlabB + 256;
static_assert(kSmem <= 232448, "shared memory budget");
static_assert(kRingA * kSlabA >= 128 * 64 * 4, "the W_UV ring holds a partial tile");
}  // namespace uvc

__global__ void __launch_bounds__(uvc::kThreads, 1) uv_combine_kernel(const __grid_constant__ UvCombineArgs a) {
  using namespace uvc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kRingA * kSlabA;
  uint64_t* a_full = reinterpret_cast<uint64_t*>(sB + kKb * kSlabB);  // [kRingA]
  uint64_t* a_empty = a_full + kRingA;                                // [kRingA]
  uint64_t* b_full = a_empty + kRingA;                                // [kKb]
  uint64_t* accum = b_full + kKb;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x, nt = blockIdx.y;
  const int ks = a.ks, nkb = kKb / ks, kb0 = static_cast<int>(blockIdx.z) * nkb, kb1 = kb0 + nkb;  // this CTA's K blocks

  if (threadIdx.x == 0) {
    for (int k = 0; k < kRingA; ++k) {
      mbar_init(&a_full[k], 1);
      mbar_init(&a_empty[k], 1);
    }
    for (int k = 0; k < kKb; ++k) mbar_init(&b_full[k], kCombWarps);  // one arrival per combine warp (own blocks)
    mbar_init(accum, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&a.mapA);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wc{a.status, abort_flag};
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 0) {
    // ---- the head's W_UV block: a weight, independent of earlier kernels,
    // so it streams while the attention drains
    if (elect_one()) {
      const uint64_t pol = policy_evict_first();
      int issued = 0;
      for (int k = 0; k < nkb; ++k, ++issued) {
        const int r = k % kRingA;
        if (!mbar_wait(&a_empty[r], ((k / kRingA) & 1) ^ 1, wc)) break;
        mbar_arrive_expect_tx(&a_full[r], kSlabA);
        tma_load_2d(sA + r * kSlabA, &a.mapA, &a_full[r], (kb0 + k) * 64, head * 128, pol);
      }
      drain_ring(a_full, kRingA, issued);  // every load has landed before the CTA may leave
    }
  } else if (warp == 1) {
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_bf16(128, 64, false, false);
      for (int k = 0; k < nkb; ++k) {
        const int r = k % kRingA;
        if (!mbar_wait(&a_full[r], (k / kRingA) & 1, wc) || !mbar_wait(&b_full[kb0 + k], 0, wc)) break;
        tc_fence_after();
        const uint32_t ab = smem_u32(sA + r * kSlabA), bb = smem_u32(sB + (kb0 + k) * kSlabB);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem, sdesc_sw128(ab + kk * 32, 16, 1024), sdesc_sw128(bb + kk * 32, 16, 1024), idesc,
                 (k | kk) ? 1u : 0u);
        mma_commit(&a_empty[r]);  // the slot takes K block k + kRingA once these MMAs retired
      }
      mma_commit(accum);  // also after an abort: the epilogue then waits only for the MMAs issued
    }
  } else {
    // ---- combine: thread t takes token nl = t / kTPR of the tile and the
    // kCPT columns [kCPT q, kCPT q + kCPT) of every 64-column K block (q = t % kTPR)
    griddep_wait();  // the partials come from the attention kernel
    const int t = threadIdx.x - 64;
    const int nl = t / kTPR, q = t % kTPR;
    const int n = nt * 64 + nl;
    int s0 = 0, s1 = 0;
    float M = -INFINITY, inv = 0.f;
    if (n < a.N) {
      s0 = a.seg_start[n];
      s1 = a.seg_start[n + 1];
      // (m, l) of the first kMl pieces in registers, their loads in flight
      // together; the rest (long sequences) from memory.  Same max, and the
      // same sum in piece order, as one loop over the pieces.
      constexpr int kMl = 8;
      float2 ml[kMl];
#pragma unroll
      for (int j = 0; j < kMl; ++j)
        ml[j] = s0 + j < s1 ? *reinterpret_cast<const float2*>(a.ml_part + (static_cast<long long>(s0 + j) * a.n_h + head) * 2)
                            : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int j = 0; j < kMl; ++j) M = fmaxf(M, ml[j].x);
      for (int s = s0 + kMl; s < s1; ++s) M = fmaxf(M, a.ml_part[(static_cast<long long>(s) * a.n_h + head) * 2]);
      float Ls = 0.f;
#pragma unroll
      for (int j = 0; j < kMl; ++j)
        if (s0 + j < s1) Ls += exp2f(ml[j].x - M) * ml[j].y;
      for (int s = s0 + kMl; s < s1; ++s) {
        const long long i = (static_cast<long long>(s) * a.n_h + head) * 2;
        Ls += exp2f(a.ml_part[i] - M) * a.ml_part[i + 1];
      }
      inv = 1.f / Ls;
    }
    __nv_bfloat16* orow = a.olat + (static_cast<long long>(n) * a.n_h + head) * 512;
    auto pass = [&](auto nj, int k) {
      constexpr int NJ = decltype(nj)::value;
      float4 acc[NJ][kF4];
#pragma unroll
      for (int j = 0; j < NJ; ++j)
#pragma unroll
        for (int i = 0; i < kF4; ++i) acc[j][i] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sb = s0; sb < s1; sb += kUnroll) {
        float wgt[kUnroll];
        float4 v[kUnroll][NJ][kF4];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const bool on = sb + u < s1;
          wgt[u] = on ? exp2f(a.ml_part[(static_cast<long long>(sb + u) * a.n_h + head) * 2] - M) : 0.f;
          const float4* src =
              reinterpret_cast<const float4*>(a.o_part + (static_cast<long long>(sb + u) * a.n_h + head) * 512);
#pragma unroll
          for (int j = 0; j < NJ; ++j)
#pragma unroll
            for (int i = 0; i < kF4; ++i)
              v[u][j][i] = on ? __ldcs(src + ((k + j) * 64 + kCPT * q) / 4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
#pragma unroll
          for (int j = 0; j < NJ; ++j)
#pragma unroll
            for (int i = 0; i < kF4; ++i) {
              acc[j][i].x += wgt[u] * v[u][j][i].x;
              acc[j][i].y += wgt[u] * v[u][j][i].y;
              acc[j][i].z += wgt[u] * v[u][j][i].z;
              acc[j][i].w += wgt[u] * v[u][j][i].w;
            }
      }
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        // row nl of K block k + j: the kCPT / 8 16-byte pieces from kCPT q / 8 on, swizzled by the row
        uint8_t* row = sB + (k + j) * kSlabB + nl * 128;
        uint4* dst = reinterpret_cast<uint4*>(orow + (k + j) * 64 + kCPT * q);
#pragma unroll
        for (int pc = 0; pc < kCPT / 8; ++pc) {
          uint32_t pk[4];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const float4 f = acc[j][2 * pc + i];
            const __nv_bfloat162 lo = __floats2bfloat162_rn(f.x * inv, f.y * inv);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(f.z * inv, f.w * inv);
            pk[2 * i] = *reinterpret_cast<const uint32_t*>(&lo);
            pk[2 * i + 1] = *reinterpret_cast<const uint32_t*>(&hi);
          }
          const uint4 pv = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(row + (((kCPT / 8 * q + pc) ^ (nl & 7)) << 4)) = pv;
          if (n < a.N) dst[pc] = pv;
        }
      }
      fence_proxy_async_smem();  // the MMAs read the tile through the async proxy
      __syncwarp();
      if (lane == 0)
#pragma unroll
        for (int j = 0; j < NJ; ++j) mbar_arrive(&b_full[k + j]);
    };
    // K blocks [kb0, kb1) in passes of kKbPass blocks, or one pass of two
    static_assert(kKbPass == 4 && kKb / kMaxKs == 2, "passes of the K splits");
    if (nkb >= kKbPass) {
      for (int k = kb0; k < kb1; k += kKbPass) pass(std::integral_constant<int, kKbPass>{}, k);
    } else {
      pass(std::integral_constant<int, 2>{}, kb0);
    }
    if (warp < 6) {
      // ---- epilogue: warps 2..5, thread <-> TMEM lane (row m of W_UV_i)
      const int q4 = warp & 3;
      const int row = q4 * 32 + lane;
      const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
      mbar_wait(accum, 0, wc);
      tc_fence_after();
      named_bar_sync(1, 128);  // every epilogue thread sees the same abort decision
      if (!*abort_flag && ks > 1) {
        // this split's partial tile into the idle W_UV ring, [16 column
        // groups][128 rows][4] fp32; the cluster reduction below reads it
        float4* my = reinterpret_cast<float4*>(sA);
#pragma unroll 1
        for (int c = 0; c < 64; c += 16) {
          float v[16];
          tmem_ld16(trow + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < 4; ++g)
            my[((c >> 2) + g) * 128 + row] = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
        }
      } else if (!*abort_flag) {
        uint8_t* stage = sA;   // every MMA retired: the A tiles are free
#pragma unroll 1
        for (int c = 0; c < 64; c += 16) {
          float v[16];
          tmem_ld16(trow + c, v);
          tmem_wait_ld();
          epi_stage<16>(a.epi, nt * 64 + c, a.N, v, stage, c, row);
        }
        named_bar_sync(1, 128);
        epi_flush(a.epi, a.tok, 0, 128, nt * 64, 64, a.N, head, stage, threadIdx.x - 64, 128, a.status);
      }
    }
  }
  __syncwarp();
  __syncthreads();
  if (ks > 1) {
    // ---- split-K reduction across the cluster (every CTA takes both
    // barriers, aborted or not, so none waits for a CTA that left)
    cluster_sync();  // every partial tile is in its CTA's shared memory
    if (warp >= 2 && warp < 6 && !*abort_flag) {
      const int z = static_cast<int>(cluster_ctarank());
      const int nr = 128 / ks, r0 = z * nr;
      const int tid = threadIdx.x - 64;
      uint8_t* stage = sB;  // every MMA retired: the B tiles are free
      const uint32_t part = smem_u32(sA);
      for (int u = tid; u < 16 * nr; u += 128) {
        const int cg = u / nr, row = r0 + u % nr;
        float4 p[kMaxKs];
#pragma unroll
        for (int q = 0; q < kMaxKs; ++q)
          if (q < ks) p[q] = ld_shared_cluster_v4(mapa(part + (cg * 128 + row) * 16, static_cast<uint32_t>(q)));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < kMaxKs; ++q)
          if (q < ks) {
            acc.x += p[q].x;
            acc.y += p[q].y;
            acc.z += p[q].z;
            acc.w += p[q].w;
          }
        const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
        epi_stage<4>(a.epi, nt * 64 + 4 * cg, a.N, vals, stage, 4 * cg, row);
      }
      named_bar_sync(1, 128);
      epi_flush(a.epi, a.tok, 0, 128, nt * 64, 64, a.N, head, stage, tid, 128, a.status, r0, r0 + nr);
    }
    cluster_sync();  // no CTA reads another's shared memory any more
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

}  // namespace mla
