// simt.cuh -- CUDA-core kernels of the MLA path.  They serve fp32 storage
// only (small layers such as the tiny preset, where tensor cores would need
// tf32 and the work is a few kFLOP); bf16 storage always runs on the
// tensor-core kernels.  Also here: the device-side split planner and the
// split-combine, shared by all attention kernels.
#pragma once
#include "epilogue.cuh"

namespace mla {

constexpr int kMaxSegSimt = 4;

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// ---------------------------------------------------------------- GEMM
// y[m, n] = sum_k A[head*a_hoff + m*a_sm + k*a_sk] * X[head*x_hoff + n*x_sn + k]
// Block: 32 x 8 threads, threadIdx.x -> m (so the RoPE partner m^1 is a lane
// shuffle away), threadIdx.y -> n.
struct SimtGemmArgs {
  const void* A[kMaxSegSimt];
  int seg_row0[kMaxSegSimt + 1];   // cumulative rows of the segments (dense mode)
  long long a_sm, a_sk, a_hoff;    // element strides of A (per-head offset)
  const void* X;
  long long x_sn, x_hoff;
  int M, N, K, nseg, heads;
  Epi epi[kMaxSegSimt];
  TokenMap tok;
  int* status;
};

template <typename T>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const __grid_constant__ SimtGemmArgs a) {
  const int m_all = blockIdx.x * 32 + threadIdx.x;
  const int n = blockIdx.y * 8 + threadIdx.y;
  const int head = blockIdx.z;
  int seg = 0;
  while (seg + 1 < a.nseg && m_all >= a.seg_row0[seg + 1]) ++seg;
  const int m = m_all - a.seg_row0[seg];
  const bool valid = (m_all < a.M) && (n < a.N);
  float acc = 0.f;
  if (valid) {
    const T* A = reinterpret_cast<const T*>(a.A[seg]) + head * a.a_hoff + m * a.a_sm;
    const T* X = reinterpret_cast<const T*>(a.X) + head * a.x_hoff + static_cast<long long>(n) * a.x_sn;
    for (int k = 0; k < a.K; ++k) acc += to_f32(A[k * a.a_sk]) * to_f32(X[k]);
  }
  const float partner = __shfl_xor_sync(0xffffffffu, acc, 1);
  if (valid) {
    const Epi& e = a.epi[seg];
    epi_apply<T>(e, a.tok, m, n, head, acc, partner, epi_inv_freq(e, a.tok, m), a.status);
  }
}

// ---------------------------------------------------------------- planner
// Splits the attention work of a decode batch into contiguous ranges of tiles
// (`tile_tokens` tokens of one sequence each), one range per worker.  With T
// tiles in all, the first We = min(W, T) workers each get at least one tile
// and the rest none, so every worker counted for a sequence really writes its
// partial slot.  Outputs, for every sequence b: tile_start[b] (cumulative
// tiles, [B+1]) and seg_start[b] (cumulative number of (worker, sequence)
// pieces, [B+1]).  The piece of worker w on sequence b is partial slot
// seg_start[b] + w - worker_of(tile_start[b]).
__host__ __device__ __forceinline__ int worker_of_tile(long long t, long long T, int W) {
  return static_cast<int>(((t + 1) * W + T - 1) / T) - 1;
}
__host__ __device__ __forceinline__ long long worker_begin(int w, long long T, int W) {
  return (static_cast<long long>(w) * T) / W;
}

// Inclusive scan of v over a 1024-thread block (shuffles within each warp,
// then the 32 warp totals in warp 0); `total` is the block's sum.  Every
// thread calls it; it leaves `warp_tot` free for the next call.
__device__ __forceinline__ long long block_scan_1024(long long v, long long* warp_tot, long long& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[wid] = v;
  __syncthreads();
  if (wid == 0) {
    long long t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long n = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += n;
    }
    warp_tot[lane] = t;
  }
  __syncthreads();
  if (wid > 0) v += warp_tot[wid - 1];
  total = warp_tot[31];
  __syncthreads();
  return v;
}

// Also fills the call's RoPE (cos, sin) table for the B new tokens (at
// positions seqlen[b]) when `rope` is not null, one launch fewer per step.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* seqlen, int B, int tile_tokens, int W,
                                                    int* tile_start, int* seg_start, int* status, const TokenMap tk,
                                                    float2* rope) {
  __shared__ long long s_warp[32];
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
  if (rope) {
    const int half = tk.d_R >> 1;
    for (int idx = threadIdx.x; idx < B * half; idx += 1024) {
      float c, s;
      rope_cos_sin(tok_pos(tk, idx / half), rope_inv_freq(tk, idx % half), c, s);
      rope[idx] = make_float2(c, s);
    }
  }
  // pass 1: cumulative tiles
  long long base = 0;
  for (int b0 = 0; b0 < B; b0 += 1024) {
    const int b = b0 + threadIdx.x;
    long long v = 0;
    if (b < B) {
      const int L = seqlen[b];
      if (L < 0) atomicOr(status, FAULT_PLAN);
      v = (max(L, 0) + 1 + tile_tokens - 1) / tile_tokens;
    }
    long long total;
    v = block_scan_1024(v, s_warp, total);
    if (b < B) tile_start[b + 1] = static_cast<int>(base + v);
    base += total;
  }
  if (threadIdx.x == 0) tile_start[0] = 0;
  const long long T = base;
  const int We = static_cast<int>(T < W ? T : W);  // workers that get tiles
  __syncthreads();  // tile_start written before pass 2 reads it
  // pass 2: pieces per sequence
  base = 0;
  for (int b0 = 0; b0 < B; b0 += 1024) {
    const int b = b0 + threadIdx.x;
    long long v = 0;
    if (b < B) {
      const long long t0 = (b == 0) ? 0 : tile_start[b];
      const long long t1 = tile_start[b + 1];
      v = worker_of_tile(t1 - 1, T, We) - worker_of_tile(t0, T, We) + 1;
    }
    long long total;
    v = block_scan_1024(v, s_warp, total);
    if (b < B) seg_start[b + 1] = static_cast<int>(base + v);
    base += total;
  }
  if (threadIdx.x == 0) seg_start[0] = 0;
}

// One piece of a worker's range: sequence b, tiles [t0, t1) of that sequence
// (sequence-local tile indices), partial slot `slot`.
struct Piece {
  int b, t0, t1, slot;
};

// Pieces of worker w, in order.  Calls f(piece) for each.  Host-callable too
// (the kernels pass device lambdas; a host check passes host ones).
#pragma nv_exec_check_disable
template <typename F>
__host__ __device__ __forceinline__ void for_each_piece(int w, int W, int B, const int* tile_start, const int* seg_start, F&& f) {
  const long long T = tile_start[B];
  if (T <= 0) return;
  const int We = static_cast<int>(T < W ? T : W);
  if (w >= We) return;
  const long long r0 = worker_begin(w, T, We), r1 = worker_begin(w + 1, T, We);
  if (r0 >= r1) return;
  int lo = 0, hi = B - 1;  // first b with tile_start[b+1] > r0
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (tile_start[mid + 1] > r0) hi = mid; else lo = mid + 1;
  }
  for (int b = lo; b < B && tile_start[b] < r1; ++b) {
    const long long s0 = tile_start[b], s1 = tile_start[b + 1];
    Piece p;
    p.b = b;
    p.t0 = static_cast<int>(max(r0, s0) - s0);
    p.t1 = static_cast<int>(min(r1, s1) - s0);
    p.slot = seg_start[b] + (w - worker_of_tile(s0, T, We));
    f(p);
  }
}

// ---------------------------------------------------------------- decode attention (CUDA cores)
// One CTA per (worker, head); 4 warps split the tokens of each piece.  Scores
// are in log2 units: Q_lat is pre-multiplied by log2(e)/sqrt(d_h + d_R).
// Output per piece: unnormalised O = sum_j 2^(s_j - m) c_j, with m and
// l = sum_j 2^(s_j - m).
template <typename T>
__global__ void __launch_bounds__(128) simt_decode_attn_kernel(
    const T* __restrict__ qlat, const T* __restrict__ cache, const CacheLayout lay,
    const int32_t* __restrict__ seqlen, const int* tile_start, const int* seg_start, int B, int W, int n_h,
    int d_c, int d_R, int tile_tokens, float* __restrict__ o_part, float* __restrict__ ml_part) {
  extern __shared__ float sm[];
  const int row = d_c + d_R;
  float* q = sm;                       // [row]
  float* wo = sm + row;                // [4][d_c]
  float* wml = wo + 4 * d_c;           // [4][2]
  const int w = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for_each_piece(w, W, B, tile_start, seg_start, [&](const Piece& p) {
    __syncthreads();
    for (int i = threadIdx.x; i < row; i += 128)
      q[i] = to_f32(qlat[(static_cast<long long>(p.b) * n_h + h) * row + i]);
    __syncthreads();
    const int L1 = seqlen[p.b] + 1;
    const int j0 = p.t0 * tile_tokens, j1 = min(L1, p.t1 * tile_tokens);
    float m = -INFINITY, l = 0.f;
    float o[16];
    const int per = (d_c + 31) / 32;
    for (int i = 0; i < 16; ++i) o[i] = 0.f;
    for (int j = j0 + warp; j < j1; j += 4) {
      const long long rj = lay.row(p.b, j);
      if (rj < 0) continue;  // no page for this position (reported by the call's cache write)
      const T* r = cache + rj * row;
      float s = 0.f;
      for (int i = lane; i < row; i += 32) s += q[i] * to_f32(r[i]);
      for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      const float mn = fmaxf(m, s);
      const float alpha = exp2f(m - mn);
      const float pj = exp2f(s - mn);
      l = l * alpha + pj;
      for (int i = 0; i < per && i < 16; ++i) {
        const int c = lane + 32 * i;
        o[i] = o[i] * alpha + (c < d_c ? pj * to_f32(r[c]) : 0.f);
      }
      m = mn;
    }
    for (int i = 0; i < per && i < 16; ++i) {
      const int c = lane + 32 * i;
      if (c < d_c) wo[warp * d_c + c] = o[i];
    }
    if (lane == 0) {
      wml[warp * 2] = m;
      wml[warp * 2 + 1] = l;
    }
    __syncthreads();
    float M = -INFINITY;
    for (int k = 0; k < 4; ++k) M = fmaxf(M, wml[2 * k]);
    float sc[4], Lsum = 0.f;
    for (int k = 0; k < 4; ++k) {
      sc[k] = (wml[2 * k] == -INFINITY) ? 0.f : exp2f(wml[2 * k] - M);
      Lsum += sc[k] * wml[2 * k + 1];
    }
    float* op = o_part + (static_cast<long long>(p.slot) * n_h + h) * d_c;
    for (int c = threadIdx.x; c < d_c; c += 128) {
      float acc = 0.f;
      for (int k = 0; k < 4; ++k) acc += sc[k] * wo[k * d_c + c];
      op[c] = acc;
    }
    if (threadIdx.x == 0) {
      ml_part[(static_cast<long long>(p.slot) * n_h + h) * 2] = M;
      ml_part[(static_cast<long long>(p.slot) * n_h + h) * 2 + 1] = Lsum;
    }
  });
}

// ---------------------------------------------------------------- latent RMSNorm
// RMSNorm after the compressed latents ("DeepSeek-V2 summary" (7shi.hateblo.jp)
// §3.1.2), one block per token: c^KV, as the down-projection left it in fp32,
// becomes x / sqrt(mean(x^2) + eps) * g_kv in the token's cache row, and c^Q
// likewise with g_q becomes the input of the query up-projection.
constexpr float kRmsEps = 1e-6f;

__device__ __forceinline__ float block_sum_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();  // red may still be read by the previous call
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) t += red[i];
  return t;
}

__device__ __forceinline__ float block_max_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) t = fmaxf(t, red[i]);
  return t;
}

// Finishes the latents of one token per block: the RMSNorm of c^KV (with
// g_kv) and its store into the cache row, as the storage dtype or as an E4M3
// row with its scale exponent; the RMSNorm of c^Q (with g_q).
template <typename T>
__global__ void __launch_bounds__(256) latent_norm_kernel(const float* __restrict__ ckv, const T* __restrict__ g_kv,
                                                          const float* __restrict__ cq, const T* __restrict__ g_q,
                                                          int d_cq, T* __restrict__ cq_out, const TokenMap tk,
                                                          int* status) {
  __shared__ float red[8];
  __shared__ long long s_row;
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
  const int n = blockIdx.x;
  if (g_kv || tk.fp8) {
    const float* x = ckv + static_cast<long long>(n) * tk.d_c;
    float inv = 1.f;
    if (g_kv) {
      float ss = 0.f;
      for (int c = threadIdx.x; c < tk.d_c; c += 256) ss += x[c] * x[c];
      inv = rsqrtf(block_sum_256(ss, red) / tk.d_c + kRmsEps);
    }
    if (threadIdx.x == 0) s_row = cache_row(tk, n, status);
    __syncthreads();
    if (s_row >= 0) {
      uint8_t* rowp = static_cast<uint8_t*>(tk.cache) + s_row * tk.row_bytes;
      if (!tk.fp8) {
        T* dst = reinterpret_cast<T*>(rowp);
        for (int c = threadIdx.x; c < tk.d_c; c += 256)
          dst[c] = static_cast<T>(g_kv ? x[c] * inv * to_f32(g_kv[c]) : x[c]);
      } else {
        // E4M3 row: scale exponent k = the smallest integer with amax / 2^k <= 448
        // (amax = max |c|; frexp gives amax = f 2^e, f in [0.5, 1), and
        // amax <= 448 2^k  <=>  k >= e - 9 + (f > 0.875)), codes = RNE(c / 2^k)
        float am = 0.f;
        for (int c = threadIdx.x; c < tk.d_c; c += 256) am = fmaxf(am, fabsf(g_kv ? x[c] * inv * to_f32(g_kv[c]) : x[c]));
        am = block_max_256(am, red);
        int k = 0;
        if (am > 0.f) {
          int e;
          const float f = frexpf(am, &e);
          k = e - 9 + (f > 0.875f ? 1 : 0);
        }
        const float descale = ldexpf(1.f, -k);
        for (int c = 2 * threadIdx.x; c < tk.d_c; c += 512) {
          float v0 = x[c], v1 = x[c + 1];
          if (g_kv) {
            v0 = v0 * inv * to_f32(g_kv[c]);
            v1 = v1 * inv * to_f32(g_kv[c + 1]);
          }
          const __nv_fp8x2_storage_t q = __nv_cvt_float2_to_fp8x2(make_float2(v0 * descale, v1 * descale), __NV_SATFINITE, __NV_E4M3);
          *reinterpret_cast<__nv_fp8x2_storage_t*>(rowp + c) = q;
        }
        // scale byte, then zeros to the end of the row (16 bytes after k^R)
        const int sb = tk.kr_off + 2 * tk.d_R;
        if (threadIdx.x < 16) rowp[sb + threadIdx.x] = threadIdx.x == 0 ? static_cast<uint8_t>(static_cast<int8_t>(k)) : 0;
      }
    }
  }
  if (g_q) {
    const float* x = cq + static_cast<long long>(n) * d_cq;
    float ss = 0.f;
    for (int c = threadIdx.x; c < d_cq; c += 256) ss += x[c] * x[c];
    const float inv = rsqrtf(block_sum_256(ss, red) / d_cq + kRmsEps);
    T* dst = cq_out + static_cast<long long>(n) * d_cq;
    for (int c = threadIdx.x; c < d_cq; c += 256) dst[c] = static_cast<T>(x[c] * inv * to_f32(g_q[c]));
  }
}

// ---------------------------------------------------------------- split combine
// O_lat[b][h][c] = sum_s 2^(m_s - M) O_s[c] / sum_s 2^(m_s - M) l_s over the
// pieces s of sequence b (the log-sum-exp merge of softmax partials).
template <typename T>
__device__ __forceinline__ void store4(T* dst, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* dst, float4 v) {
  *reinterpret_cast<float4*>(dst) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst, float4 v) {
  const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  *reinterpret_cast<uint2*>(dst) = make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
}

// One warp per (sequence, head): lane l owns columns 4l + 128k.  The pieces
// are merged in order, weights 2^(m_s - M), then normalised by the merged l.
// The weights of up to kCombineUnroll pieces are formed first, so that all
// of a lane's partial loads of a column group are in flight together.
constexpr int kCombineUnroll = 4;

template <typename T>
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ o_part, const float* __restrict__ ml_part,
                                                     const int* seg_start, int n_h, int d_c, T* __restrict__ olat) {
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
  const int b = blockIdx.x, h = blockIdx.y * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (h >= n_h) return;
  const int s0 = seg_start[b], s1 = seg_start[b + 1];
  float M = -INFINITY;
  for (int s = s0; s < s1; ++s) M = fmaxf(M, ml_part[(static_cast<long long>(s) * n_h + h) * 2]);
  float Ls = 0.f;
  for (int s = s0; s < s1; ++s) {
    const long long i = (static_cast<long long>(s) * n_h + h) * 2;
    Ls += exp2f(ml_part[i] - M) * ml_part[i + 1];
  }
  const float inv = 1.f / Ls;
  float4 acc[4];  // columns lane * 4 + 128 k, k < d_c / 128 (d_c <= 512)
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int nk = lane * 4 < d_c ? (d_c - lane * 4 + 127) / 128 : 0;  // this lane's column groups
  for (int sb = s0; sb < s1; sb += kCombineUnroll) {
    float wgt[kCombineUnroll];
#pragma unroll
    for (int u = 0; u < kCombineUnroll; ++u)
      wgt[u] = sb + u < s1 ? exp2f(ml_part[(static_cast<long long>(sb + u) * n_h + h) * 2] - M) : 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k >= nk) break;
      float4 v[kCombineUnroll];
#pragma unroll
      for (int u = 0; u < kCombineUnroll; ++u)
        v[u] = sb + u < s1 ? __ldcs(reinterpret_cast<const float4*>(
                                 o_part + (static_cast<long long>(sb + u) * n_h + h) * d_c + lane * 4 + 128 * k))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < kCombineUnroll; ++u) {
        acc[k].x += wgt[u] * v[u].x; acc[k].y += wgt[u] * v[u].y;
        acc[k].z += wgt[u] * v[u].z; acc[k].w += wgt[u] * v[u].w;
      }
    }
  }
  for (int k = 0; k < nk; ++k)
    store4<T>(olat + (static_cast<long long>(b) * n_h + h) * d_c + lane * 4 + 128 * k,
              make_float4(acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv));
}

// ---------------------------------------------------------------- prefill attention (CUDA cores)
// Un-absorbed causal attention for token t (position start_pos + t) and head h:
//   s_j = [q^C; q^R] . [K^C_j; k^R_j]  (log2 units, q pre-scaled), j = 0..start_pos+t
//   o   = sum_j softmax(s)_j V_j
// qp: [T][n_h][d_h + d_R]; kc, v: [start_pos + T][n_h][d_h]; k^R from the cache rows.
template <typename T>
__global__ void __launch_bounds__(128) simt_prefill_attn_kernel(
    const T* __restrict__ qp, const T* __restrict__ kc, const T* __restrict__ vv, const T* __restrict__ cache_seq,
    int T_new, int start_pos, int n_h, int d_h, int d_R, int d_c, T* __restrict__ out) {
  extern __shared__ float sm[];
  const int dq = d_h + d_R;
  float* q = sm;              // [dq]
  float* wo = sm + dq;        // [4][d_h]
  float* wml = wo + 4 * d_h;  // [4][2]
  const int t = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < dq; i += 128) q[i] = to_f32(qp[(static_cast<long long>(t) * n_h + h) * dq + i]);
  __syncthreads();
  const int nkeys = start_pos + t + 1;
  const int row = d_c + d_R;
  float m = -INFINITY, l = 0.f;
  float o[8];
  for (int i = 0; i < 8; ++i) o[i] = 0.f;
  for (int j = warp; j < nkeys; j += 4) {
    const T* kj = kc + (static_cast<long long>(j) * n_h + h) * d_h;
    const T* kr = cache_seq + static_cast<long long>(j) * row + d_c;
    float s = 0.f;
    for (int i = lane; i < d_h; i += 32) s += q[i] * to_f32(kj[i]);
    for (int i = lane; i < d_R; i += 32) s += q[d_h + i] * to_f32(kr[i]);
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float mn = fmaxf(m, s);
    const float alpha = exp2f(m - mn), pj = exp2f(s - mn);
    l = l * alpha + pj;
    const T* vj = vv + (static_cast<long long>(j) * n_h + h) * d_h;
    for (int i = 0; i < 8; ++i) {
      const int c = lane + 32 * i;
      o[i] = o[i] * alpha + (c < d_h ? pj * to_f32(vj[c]) : 0.f);
    }
    m = mn;
  }
  for (int i = 0; i < 8; ++i) {
    const int c = lane + 32 * i;
    if (c < d_h) wo[warp * d_h + c] = o[i];
  }
  if (lane == 0) { wml[2 * warp] = m; wml[2 * warp + 1] = l; }
  __syncthreads();
  float M = -INFINITY;
  for (int k = 0; k < 4; ++k) M = fmaxf(M, wml[2 * k]);
  float sc[4], Ls = 0.f;
  for (int k = 0; k < 4; ++k) {
    sc[k] = (wml[2 * k] == -INFINITY) ? 0.f : exp2f(wml[2 * k] - M);
    Ls += sc[k] * wml[2 * k + 1];
  }
  for (int c = threadIdx.x; c < d_h; c += 128) {
    float acc = 0.f;
    for (int k = 0; k < 4; ++k) acc += sc[k] * wo[k * d_h + c];
    out[(static_cast<long long>(t) * n_h + h) * d_h + c] = static_cast<T>(acc / Ls);
  }
}

}  // namespace mla
