// attn_prefill_tc.cuh -- tensor-core causal attention of the MLA prefill
// ("DeepSeek-V2 summary" (7shi.hateblo.jp), App. C, o_{t,i} = sum over j <= t),
// in the un-absorbed form: every key is formed once per token,
//   k_{j,i} = [K^C_{j,i} (d_h) ; k^R_j (d_R, shared by the heads)],  v_{j,i} = V_{j,i},
// so each (query, key) pair costs 2 (d_h + d_R) + 2 d_h flops instead of the
// 2 (d_c + d_R) + 2 d_c of the absorbed form.
//
// One CTA per (tile of 128 queries, head), d_h = 128, d_R = 64:
//   S = Q K^T      tcgen05.mma M = 128 queries, N = 128 keys, K = 192; S double-buffered in TMEM
//   P = 2^(S - m)  two threads per query row (64 keys each), lazily refreshed running max
//   O += P V       P (bf16) written back to TMEM (two buffers) and used as the A operand; V read MN-major
// Warp roles (320 threads): warp 0 TMA, warp 1 TMEM owner and MMA issuer,
// warps 2-9 softmax and epilogue.  The softmax is the kernel's longest stage
// (128 exponentials per query row and key tile), so each row is shared by two
// threads of one warp through the 16-lane TMEM access shape: thread t < 16 and
// t + 16 take the row's keys in alternate runs of 16.  Causal: key tiles 0 .. (last query)/128;
// the tiles with the most keys are launched first.
#pragma once
#include "ptx.cuh"

namespace mla {

namespace pf {
constexpr int kQ = 128, kK = 128;                 // queries / keys per tile
constexpr int kChunk = 128 * 128;                 // 128 rows x 64 columns bf16
constexpr int kQBytes = 3 * kChunk;               // Q: [128 x 192]
constexpr int kKBytes = 3 * kChunk;               // K: [128 x (128 + 64)]
constexpr int kVBytes = 2 * kChunk;               // V: [128 x 128]
constexpr int kStages = 2;
constexpr int kSmem = 1024 + kQBytes + kStages * (kKBytes + kVBytes) + 256;
// TMEM columns: O [0,128), S two buffers of 128, P two buffers of 64 (bf16 pairs)
constexpr uint32_t kTmemO = 0, kTmemS = 128, kTmemP = 384, kTmemCols = 512;
constexpr float kRescaleLog2 = 8.f;
constexpr int kThreads = 320;
constexpr int kPolyEvery = 4;  // one key pair in kPolyEvery takes its exponentials on the FMA pipe

// 2^x for x <= 128 on the FMA pipe (the softmax's exponentials are bound by
// the MUFU unit; a share of them computed here balances the two).  x = n + f
// with n = round(x) (by the 1.5 * 2^23 rounding constant) and f in [-1/2, 1/2];
// 2^f is a degree-3 polynomial fitted to 2^f on that interval (relative
// error 7.5e-5, below half a bf16 ulp), and n is added to its exponent field.
// Inputs below -126 (masked keys are -inf) give 2^-126, which P rounds to a
// bf16 that adds nothing measurable to O or l.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;
  const float f = x - (t - 12582912.f);
  const float p = fmaf(fmaf(fmaf(0.05517104f, f, 0.24261111f), f, 0.69326109f), f, 0.99992806f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}
}  // namespace pf

struct PrefillArgs {
  CUtensorMap map_q;    // Qp  [T x n_h*192]  (pre-scaled by log2(e)/sqrt(192)), box {64, 128}
  CUtensorMap map_kc;   // K^C [S x n_h*128], box {64, 128}
  CUtensorMap map_kr;   // cache rows of the sequence [S x 576]; k^R at column 512, box {64, 128}
  CUtensorMap map_v;    // V   [S x n_h*128], box {64, 128}
  __nv_bfloat16* out;   // [T][n_h][128], normalised
  int T, start_pos, n_h, n_qt;
  int* status;
};

__global__ void __launch_bounds__(pf::kThreads, 1) attn_prefill_tc_kernel(const __grid_constant__ PrefillArgs a) {
  using namespace pf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sq = smem;
  uint8_t* sk = sq + kQBytes;
  uint8_t* sv = sk + kStages * kKBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sv + kStages * kVBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;       // [2]
  uint64_t* k_empty = k_full + 2;      // [2]
  uint64_t* v_full = k_empty + 2;      // [2]
  uint64_t* v_empty = v_full + 2;      // [2]
  uint64_t* s_full = v_empty + 2;      // [2]
  uint64_t* s_free = s_full + 2;       // [2]
  uint64_t* p_full = s_free + 2;       // [2] P(j) written into P buffer j % 2
  uint64_t* p_free = p_full + 2;       // [2] PV(j) retired, P buffer j % 2 free
  uint64_t* o_done = p_free + 2;
  uint64_t* drain = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = a.n_qt - 1 - static_cast<int>(blockIdx.x);  // heaviest tiles first
  const int h = blockIdx.y;
  const int q0 = qt * kQ;
  const int q_last = min(q0 + kQ, a.T) - 1;                     // last query of the tile
  const int nk = (a.start_pos + q_last) / kK + 1;              // key tiles

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 256);  // every softmax thread
      mbar_init(&p_full[i], 256);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&a.map_q);
    prefetch_tmap(&a.map_kc);
    prefetch_tmap(&a.map_kr);
    prefetch_tmap(&a.map_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wc{a.status, abort_flag};

  if (warp == 0) {
    if (elect_one()) {
      const uint64_t keep = policy_evict_last();
      mbar_arrive_expect_tx(q_full, kQBytes);
      for (int c = 0; c < 3; ++c) tma_load_2d(sq + c * kChunk, &a.map_q, q_full, h * 192 + c * 64, q0, keep);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nk; ++j) {
        const int s = j & 1;
        const uint32_t ph = ((j >> 1) & 1) ^ 1;
        const int y = j * kK;
        if (!mbar_wait(&k_empty[s], ph, wc)) break;
        mbar_arrive_expect_tx(&k_full[s], kKBytes);
        uint8_t* kd = sk + s * kKBytes;
        tma_load_2d(kd, &a.map_kc, &k_full[s], h * 128, y, keep);
        tma_load_2d(kd + kChunk, &a.map_kc, &k_full[s], h * 128 + 64, y, keep);
        tma_load_2d(kd + 2 * kChunk, &a.map_kr, &k_full[s], 512, y, keep);
        ++k_issued;
        if (!mbar_wait(&v_empty[s], ph, wc)) break;
        mbar_arrive_expect_tx(&v_full[s], kVBytes);
        uint8_t* vd = sv + s * kVBytes;
        tma_load_2d(vd, &a.map_v, &v_full[s], h * 128, y, keep);
        tma_load_2d(vd + kChunk, &a.map_v, &v_full[s], h * 128 + 64, y, keep);
        ++v_issued;
      }
      // every issued load has landed before the CTA may leave
      drain_ring(q_full, 1, 1);
      drain_ring(k_full, 2, k_issued);
      drain_ring(v_full, 2, v_issued);
    }
  } else if (warp == 1) {
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 128, false, true);
      bool ok = mbar_wait(q_full, 0, wc);
      tc_fence_after();
      const uint32_t qb = smem_u32(sq);
      for (int j = 0; ok && j <= nk; ++j) {
        if (j < nk) {  // S(j) = Q K(j)^T into S buffer j&1
          const int s = j & 1;
          if (!mbar_wait(&k_full[s], (j >> 1) & 1, wc) || !mbar_wait(&s_free[s], ((j >> 1) & 1) ^ 1, wc)) break;
          tc_fence_after();
          const uint32_t kb = smem_u32(sk + s * kKBytes);
          for (int c = 0; c < 3; ++c) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem + kTmemS + s * 128, sdesc_sw128(qb + c * kChunk + kk * 32, 16, 1024),
                     sdesc_sw128(kb + c * kChunk + kk * 32, 16, 1024), idesc_s, (c | kk) ? 1u : 0u);
          }
          mma_commit(&s_full[s]);
          mma_commit(&k_empty[s]);
        }
        if (j > 0) {  // O += P(j-1) V(j-1)
          const int jj = j - 1, s = jj & 1;
          if (!mbar_wait(&p_full[s], (jj >> 1) & 1, wc) || !mbar_wait(&v_full[s], (jj >> 1) & 1, wc)) break;
          tc_fence_after();
          const uint32_t vb = smem_u32(sv + s * kVBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + kTmemO, tmem + kTmemP + s * 64 + kk * 8, sdesc_sw128(vb + kk * 2048, kChunk, 1024), idesc_pv,
                   (jj > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&p_free[s]);
          mma_commit(&v_empty[s]);
          if (j == nk) mma_commit(o_done);
        }
      }
      mma_commit(drain);
    }
  } else {
    // warp w (2..9) takes rows [32 (w % 4) + 16 sub, +16) (sub = (w - 2) / 4),
    // a TMEM lane quarter it may access; thread t its row's keys 32 c + 16 hf
    // + i (c < 4, i < 16, hf = t / 16), and the same columns of O
    const int q4 = warp & 3, sub = (warp - 2) >> 2, hf = lane >> 4;
    const int rbase = q4 * 32 + sub * 16;
    const int r = rbase + (lane & 15);            // query row of the tile = TMEM lane
    const uint32_t tl = tmem + (static_cast<uint32_t>(rbase) << 16);
    const int qpos = a.start_pos + q0 + r;        // position of this query in the sequence
    float m_run = -INFINITY, l_run = 0.f;         // l_run: this thread's keys only
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      const int s = j & 1;
      if (!mbar_wait(&s_full[s], (j >> 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld16x2(tl + kTmemS + s * 128 + c * 32, *reinterpret_cast<uint32_t(*)[16]>(&sr[c * 16]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[s]);
      const int key0 = j * kK + 16 * hf;          // key of sr[16 c + i] is key0 + 32 c + i
      float mt = -INFINITY;
      const bool diag = j * kK + kK - 1 > qpos;   // some keys of this tile lie after the query
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        float v = __uint_as_float(sr[c]);
        if (diag && key0 + 32 * (c >> 4) + (c & 15) > qpos) v = -INFINITY;
        sr[c] = __float_as_uint(v);
        mt = fmaxf(mt, v);
      }
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));  // the whole row
      float m_new = m_run, alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_new = mt;
      } else if (mt > m_run + kRescaleLog2) {
        m_new = mt;
        alpha = ex2_approx(m_run - m_new);
        rescale = true;
      }
      uint32_t pk[32];
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const bool poly = c % kPolyEvery == kPolyEvery - 1;
        const float x0 = __uint_as_float(sr[2 * c]) - m_new, x1 = __uint_as_float(sr[2 * c + 1]) - m_new;
        const float p0 = poly ? exp2_poly(x0) : ex2_approx(x0);
        const float p1 = poly ? exp2_poly(x1) : ex2_approx(x1);
        lsum += p0 + p1;
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
        pk[c] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      l_run = l_run * alpha + lsum;
      m_run = m_new;
      // P buffer j % 2 is free once PV(j-2) retired; O is settled for a
      // rescale once PV(j-1) retired too
      if (!mbar_wait(&p_free[s], ((j >> 1) & 1) ^ 1, wc)) { ok = false; break; }
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale)) {
        if (j > 0 && !mbar_wait(&p_free[s ^ 1], ((j - 1) >> 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < 128; c += 32) {
          uint32_t o[16];
          tmem_ld16x2(tl + kTmemO + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st16x2(tl + kTmemO + c, o);
        }
      }
      // P columns (bf16 pairs): keys 32 c + 16 hf + 2 i, +1 -> column 16 c + 8 hf + i
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_st16x2_x8(tl + kTmemP + s * 64 + 16 * c, *reinterpret_cast<uint32_t(*)[8]>(&pk[8 * c]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[s]);
    }
    if (ok && mbar_wait(o_done, 0, wc)) {
      tc_fence_after();
      const float inv = 1.f / (l_run + __shfl_xor_sync(0xffffffffu, l_run, 16));
      const int t = q0 + r;
      __nv_bfloat16* dst = a.out + (static_cast<long long>(t) * a.n_h + h) * 128 + 16 * hf;
      for (int c = 0; c < 128; c += 32) {
        uint32_t o[16];
        tmem_ld16x2(tl + kTmemO + c, o);
        tmem_wait_ld();
        if (t < a.T) {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            uint4 w;
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[8 * i + 2 * e]) * inv,
                                                              __uint_as_float(o[8 * i + 2 * e + 1]) * inv);
              wp[e] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            reinterpret_cast<uint4*>(dst + c)[i] = w;
          }
        }
      }
    }
  }
  if (warp == 1) {  // TMEM is freed only after every MMA retired (bounded; not cut short by an abort)
    __syncwarp();
    if (lane == 0) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(smem_u32(drain), 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  }
  __syncwarp();  // every warp reconverged (elected lanes) before the aligned barrier
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mla
