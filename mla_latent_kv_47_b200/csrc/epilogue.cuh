// epilogue.cuh -- what happens to one GEMM output element y[m, n] (feature m,
// token n) once its dot product is complete: plain stores, the decoupled RoPE
// of "DeepSeek-V2 summary" (7shi.hateblo.jp) §2.1.3 applied to q^R and k^R,
// and the cache-row writes of the boxed vectors of App. C.
#pragma once
#include "ptx.cuh"

namespace mla {

enum EpiKind : int {
  EPI_STORE = 0,       // out[n * ld + col0 + m] = y * scale
  EPI_QLAT_ROPE = 1,   // m = head * d_R + j:  Qlat[n][head][d_c + j] = RoPE(y)_j * scale
  EPI_PER_HEAD = 2,    // per-head GEMM:  out[n * ld + head * hs + m] = y * scale
  EPI_CACHE_CKV = 3,   // m = c:  cache[row(n)][c] = y
  EPI_CACHE_KR = 4,    // m = j:  cache[row(n)][d_c + j] = RoPE(y)_j
  EPI_QP_ROPE = 5,     // m = head * d_R + j:  out[n][head][d_h + j] = RoPE(y)_j * scale  (prefill q)
  EPI_HEADS = 6,       // m = head * d_h + e:  out[n][head][e] = y * scale  (row stride ld, head stride hs)
};

struct Epi {
  int kind;
  int out_f32;      // 1: fp32 output, 0: bf16 (or the storage type on the CUDA-core path)
  void* out;
  long long ld;     // elements between consecutive tokens n
  long long hs;     // elements between heads (EPI_HEADS / EPI_QP_ROPE / EPI_QLAT_*)
  int col0;         // column offset (EPI_STORE) or head-local offset (EPI_HEADS, EPI_QP_ROPE)
  int dh;           // rows per head for EPI_HEADS
  float scale;
};

// Where the cache rows of each sequence live: contiguous from seq_start[s],
// or, with a block table, in pages of block_size rows (a multiple of the
// 64-token attention tile, so a tile never straddles two pages).
struct CacheLayout {
  const int64_t* seq_start;
  const int32_t* block_table;  // NULL: contiguous; else [n_seq][max_blocks] page numbers
  int block_size, max_blocks;

  // Positions the layout can hold for one sequence (paged), else no limit.
  __device__ __forceinline__ bool holds(long long p) const {
    return !block_table || p < static_cast<long long>(max_blocks) * block_size;
  }
  // Row of position p of sequence s; negative when the block table has no
  // page for it (a position past max_blocks pages, or a negative entry).
  __device__ __forceinline__ long long row(int s, long long p) const {
    if (!block_table) return seq_start[s] + p;
    if (!holds(p)) return -1;
    const long long page = block_table[static_cast<long long>(s) * max_blocks + p / block_size];
    return page < 0 ? -1 : page * block_size + p % block_size;
  }
};

// Where token n of a GEMM sits: its sequence, its position, its cache row.
struct TokenMap {
  const int32_t* pos;        // position of token n, or NULL: pos_base + n
  int pos_base;
  const int32_t* seq;        // sequence of token n, or NULL: seq_const (>= 0) or n (seq_const < 0)
  int seq_const;
  CacheLayout lay;           // cache rows of each sequence
  const int32_t* capacity;   // NULL or rows reserved per sequence
  long long n_rows;          // rows allocated in the cache
  void* cache;
  int row_bytes;             // bytes of one cache row
  int kr_off;                // byte offset of k^R inside a row
  int fp8;                   // rows hold E4M3 c^KV (written by the latent finish kernel, not the GEMM)
  int d_c, d_R;
  double log2_base;          // log2(rope_base)
  const float2* rope;        // NULL, or (cos, sin) of pair i at token n: rope[n * d_R / 2 + i]
  double yarn_s;             // 0: plain RoPE; else the YaRN scale s (with alpha, beta, L0 below)
  double yarn_alpha, yarn_beta, yarn_L0;
};

__device__ __forceinline__ int tok_pos(const TokenMap& t, int n) { return t.pos ? t.pos[n] : t.pos_base + n; }
__device__ __forceinline__ int tok_seq(const TokenMap& t, int n) {
  return t.seq ? t.seq[n] : (t.seq_const >= 0 ? t.seq_const : n);
}

// Rotation angle of pair i at position pos, reduced to [-pi, pi].  The
// product pos * base^(-2i/d_R) is formed and reduced in fp64 (positions reach
// 1.3e5, where an fp32 angle would already be off by ~4e-3 rad), then sine and
// cosine are taken in fp32.
// Rotary frequency of pair i: theta_i = base^(-2i/d_R) (RoFormer), or with
// YaRN ("DeepSeek-V2 summary" (7shi.hateblo.jp) §3.1.4: s, alpha, beta and the
// pre-training length L0) the published YaRN rule: a pair whose wavelength
// 2 pi / theta_i fits more than beta times into L0 keeps theta_i, one that fits
// fewer than alpha times takes theta_i / s, and in between the two blend
// linearly in r = L0 theta_i / (2 pi).
__device__ __forceinline__ double rope_inv_freq(const TokenMap& t, int i) {
  const double theta = exp2(-(2.0 * i / t.d_R) * t.log2_base);
  if (!(t.yarn_s > 0.0)) return theta;
  const double r = t.yarn_L0 * theta * (1.0 / 6.283185307179586);
  const double ramp = fmin(fmax((r - t.yarn_alpha) / (t.yarn_beta - t.yarn_alpha), 0.0), 1.0);
  return (1.0 - ramp) * (theta / t.yarn_s) + ramp * theta;
}
__device__ __noinline__ void rope_cos_sin(int pos, double inv_freq, float& c, float& s) {
  const double two_pi_hi = 6.283185307179586;
  const double two_pi_lo = 2.4492935982947064e-16;
  double phi = static_cast<double>(pos) * inv_freq;
  double k = rint(phi * (1.0 / two_pi_hi));
  double r = fma(-k, two_pi_hi, phi);
  r = fma(-k, two_pi_lo, r);
  sincosf(static_cast<float>(r), &s, &c);
}

// (cos, sin) of pair i at token n: from the call's table when there is one,
// else computed here.  Both give the same bits (the table is filled by
// rope_table_kernel with rope_cos_sin).
__device__ __forceinline__ void rope_cs(const TokenMap& t, int n, int i, double inv_freq, float& c, float& s) {
  if (t.rope) {
    const float2 v = t.rope[static_cast<long long>(n) * (t.d_R >> 1) + i];
    c = v.x;
    s = v.y;
  } else {
    rope_cos_sin(tok_pos(t, n), inv_freq, c, s);
  }
}

// Rotated value of component j (of an interleaved pair) given its own value y
// and its partner's value yp: (a, b) -> (a cos - b sin, a sin + b cos).
__device__ __forceinline__ float rope_apply(int j, float y, float yp, float c, float s) {
  return (j & 1) ? (yp * s + y * c) : (y * c - yp * s);
}

template <typename T>
__device__ __forceinline__ void store_elem(void* base, long long idx, float v, int out_f32) {
  if (out_f32) {
    reinterpret_cast<float*>(base)[idx] = v;
  } else {
    reinterpret_cast<T*>(base)[idx] = static_cast<T>(v);
  }
}

// Cache row of token n or -1 when the write must be skipped (capacity).
__device__ __forceinline__ long long cache_row(const TokenMap& t, int n, int* status) {
  const int s = tok_seq(t, n);
  const int p = tok_pos(t, n);
  if (p < 0 || (t.capacity && p >= t.capacity[s]) || !t.lay.holds(p)) {
    atomicOr(status, FAULT_CAPACITY);
    return -1;
  }
  const long long row = t.lay.row(s, p);
  if (row < 0 || row >= t.n_rows) {
    atomicOr(status, FAULT_CAPACITY);
    return -1;
  }
  return row;
}

// Applies the epilogue to y = output (m, n).  `yp` is the value of the rotary
// partner (m ^ 1, n), needed by the RoPE kinds.  `head` is the batch index of
// per-head GEMMs.  T is the storage type of bf16/fp32 outputs.
template <typename T>
__device__ __forceinline__ void epi_apply(const Epi& e, const TokenMap& tk, int m, int n, int head, float y,
                                          float yp, double inv_freq, int* status) {
  switch (e.kind) {
    case EPI_STORE:
      store_elem<T>(e.out, static_cast<long long>(n) * e.ld + e.col0 + m, y * e.scale, e.out_f32);
      break;
    case EPI_QLAT_ROPE: {
      const int hh = m / tk.d_R, j = m % tk.d_R;
      float c, s;
      rope_cs(tk, n, j >> 1, inv_freq, c, s);
      const float r = rope_apply(j, y, yp, c, s);
      store_elem<T>(e.out, static_cast<long long>(n) * e.ld + hh * e.hs + tk.d_c + j, r * e.scale, e.out_f32);
      break;
    }
    case EPI_PER_HEAD:
      store_elem<T>(e.out, static_cast<long long>(n) * e.ld + head * e.hs + m, y * e.scale, e.out_f32);
      break;
    case EPI_CACHE_CKV: {
      const long long row = cache_row(tk, n, status);
      if (row >= 0) store_elem<T>(static_cast<uint8_t*>(tk.cache) + row * tk.row_bytes, m, y, 0);
      break;
    }
    case EPI_CACHE_KR: {
      const long long row = cache_row(tk, n, status);
      float c, s;
      rope_cs(tk, n, m >> 1, inv_freq, c, s);
      const float r = rope_apply(m, y, yp, c, s);
      if (row >= 0) store_elem<T>(static_cast<uint8_t*>(tk.cache) + row * tk.row_bytes + tk.kr_off, m, r, 0);
      break;
    }
    case EPI_QP_ROPE: {
      const int hh = m / tk.d_R, j = m % tk.d_R;
      float c, s;
      rope_cs(tk, n, j >> 1, inv_freq, c, s);
      const float r = rope_apply(j, y, yp, c, s);
      store_elem<T>(e.out, static_cast<long long>(n) * e.ld + hh * e.hs + e.col0 + j, r * e.scale, e.out_f32);
      break;
    }
    case EPI_HEADS: {
      const int hh = m / e.dh, j = m % e.dh;
      store_elem<T>(e.out, static_cast<long long>(n) * e.ld + hh * e.hs + e.col0 + j, y * e.scale, e.out_f32);
      break;
    }
  }
}

// ---- staged epilogue of the tensor-core GEMM.
// Phase 1 (thread = output row m of the tile): each output goes into a staging
// tile in shared memory, column-major ([n][128 rows]), so consecutive rows of
// one token sit side by side: the final value (scaled, in the output type) for
// plain kinds, the raw fp32 value for the rotary kinds.
// Phase 2 (all epilogue threads): runs of 8 rows of one token (16 bytes of
// bf16 or 32 of fp32) go to their destination with vector stores; a rotary run
// is 4 interleaved pairs, rotated here with one 32-byte load of their (cos, sin)
// from the call's table.  Every kind maps a run of 8 consecutive rows to 8
// consecutive destination elements (head blocks are multiples of 8 rows).

__device__ __forceinline__ bool epi_rotary(int kind) {
  return kind == EPI_QLAT_ROPE || kind == EPI_CACHE_KR || kind == EPI_QP_ROPE;
}

// Phase 1 for NV consecutive columns n0.. held by this thread.
template <int NV>
__device__ __forceinline__ void epi_stage(const Epi& e, int n0, int n_end, const float* v, uint8_t* stage, int nl0, int ml) {
  if (epi_rotary(e.kind) || e.out_f32) {
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const float r = epi_rotary(e.kind) ? v[j] : v[j] * e.scale;
      reinterpret_cast<float*>(stage)[(nl0 + j) * 128 + ml] = (n0 + j < n_end) ? r : 0.f;
    }
  } else {
    const float sc = e.kind == EPI_CACHE_CKV ? 1.f : e.scale;
#pragma unroll
    for (int j = 0; j < NV; ++j)
      reinterpret_cast<__nv_bfloat16*>(stage)[(nl0 + j) * 128 + ml] = __float2bfloat16_rn((n0 + j < n_end) ? v[j] * sc : 0.f);
  }
}

// Destination of the run of rows m.. (a multiple of 8) of token n, or nullptr
// when the token's cache row is out of bounds (recorded in the status word).
__device__ __forceinline__ uint8_t* epi_addr(const Epi& e, const TokenMap& tk, int m, int n, int head, int* status) {
  const int es = e.out_f32 ? 4 : 2;
  long long idx;
  switch (e.kind) {
    case EPI_QLAT_ROPE: idx = static_cast<long long>(n) * e.ld + (m / tk.d_R) * e.hs + tk.d_c + m % tk.d_R; break;
    case EPI_QP_ROPE: idx = static_cast<long long>(n) * e.ld + (m / tk.d_R) * e.hs + e.col0 + m % tk.d_R; break;
    case EPI_HEADS: idx = static_cast<long long>(n) * e.ld + (m / e.dh) * e.hs + e.col0 + m % e.dh; break;
    case EPI_PER_HEAD: idx = static_cast<long long>(n) * e.ld + head * e.hs + m; break;
    case EPI_CACHE_CKV:
    case EPI_CACHE_KR: {
      const long long row = cache_row(tk, n, status);
      if (row < 0) return nullptr;
      return static_cast<uint8_t*>(tk.cache) + row * tk.row_bytes + (e.kind == EPI_CACHE_KR ? tk.kr_off : 0) + m * 2;
    }
    default: idx = static_cast<long long>(n) * e.ld + e.col0 + m; break;
  }
  return static_cast<uint8_t*>(e.out) + idx * es;
}

// Rotated, scaled run of 8 rows (4 interleaved pairs starting at pair i0) of
// token n from the fp32 staging tile.
__device__ __forceinline__ void epi_rope_run(const Epi& e, const TokenMap& tk, int n, int i0, const float* x, float* y) {
  float c[4], s[4];
  if (tk.rope) {
    const float4* t = reinterpret_cast<const float4*>(tk.rope + static_cast<long long>(n) * (tk.d_R >> 1) + i0);
    const float4 a = t[0], b = t[1];
    c[0] = a.x; s[0] = a.y; c[1] = a.z; s[1] = a.w; c[2] = b.x; s[2] = b.y; c[3] = b.z; s[3] = b.w;
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) rope_cos_sin(tok_pos(tk, n), rope_inv_freq(tk, i0 + q), c[q], s[q]);
  }
  const float sc = e.kind == EPI_CACHE_KR ? 1.f : e.scale;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    y[2 * q] = (x[2 * q] * c[q] - x[2 * q + 1] * s[q]) * sc;
    y[2 * q + 1] = (x[2 * q] * s[q] + x[2 * q + 1] * c[q]) * sc;
  }
}

// Phase 2: the staged tile (tokens n_base .. n_base + n_cols - 1, rows m0 ..
// m0 + 127) to global memory; thread tid of nthr.  Plain kinds take a direct
// path (destination of a token computed once, loop unrolled so the
// shared-memory loads and global stores overlap); cache and rotary kinds take
// the general one.
__device__ __forceinline__ void epi_flush(const Epi& e, const TokenMap& tk, int m0, int rows_valid, int n_base, int n_cols,
                                          int n_end, int head, const uint8_t* stage, int tid, int nthr, int* status,
                                          int ml_lo = 0, int ml_hi = 128) {
  // only the tile rows [ml_lo, ml_hi) (multiples of 8) are written
  const int kind = e.kind;
  const bool rot = epi_rotary(kind);
  if (!rot && kind != EPI_CACHE_CKV) {
    // runs of 16 bytes: 8 bf16 or 4 fp32 rows
    const int es = e.out_f32 ? 4 : 2;
    uint8_t* const out = static_cast<uint8_t*>(e.out);
    const long long ld = e.ld;
    const long long off0 = kind == EPI_PER_HEAD ? static_cast<long long>(head) * e.hs : e.col0;
    const int lg_lo = __ffs(((ml_hi - ml_lo) / (16 / es))) - 1;  // log2 of runs per token in the row range
    const int total = n_cols << lg_lo;
#pragma unroll 4
    for (int id = tid; id < total; id += nthr) {
      const int nl = id >> lg_lo, ml = ml_lo + (id & ((1 << lg_lo) - 1)) * (16 / es);
      const int n = n_base + nl, m = m0 + ml;
      if (n >= n_end || m >= rows_valid) continue;
      long long idx;
      if (kind == EPI_HEADS) idx = static_cast<long long>(n) * ld + (m / e.dh) * e.hs + e.col0 + m % e.dh;
      else idx = static_cast<long long>(n) * ld + off0 + m;
      *reinterpret_cast<uint4*>(out + idx * es) = *reinterpret_cast<const uint4*>(stage + (nl * 128 + ml) * es);
    }
    return;
  }
  const bool f32 = rot || e.out_f32;  // staging type
  const int vec = (!rot && e.out_f32) ? 4 : 8;  // rows per run
  const int runs = (ml_hi - ml_lo) / vec;
  for (int id = tid; id < n_cols * runs; id += nthr) {
    const int nl = id / runs, ml = ml_lo + (id % runs) * vec;
    const int n = n_base + nl, m = m0 + ml;
    if (n >= n_end || m >= rows_valid) continue;
    uint8_t* dst = epi_addr(e, tk, m, n, head, status);
    if (!dst) continue;
    if (rot) {
      const float4* src = reinterpret_cast<const float4*>(stage + (nl * 128 + ml) * 4);
      const float4 a = src[0], b = src[1];
      const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      float y[8];
      const int i0 = (kind == EPI_CACHE_KR ? m : m % tk.d_R) >> 1;
      epi_rope_run(e, tk, n, i0, x, y);
      if (e.out_f32) {
        reinterpret_cast<float4*>(dst)[0] = make_float4(y[0], y[1], y[2], y[3]);
        reinterpret_cast<float4*>(dst)[1] = make_float4(y[4], y[5], y[6], y[7]);
      } else {
        uint4 o;
        __nv_bfloat162 t;
        t = __floats2bfloat162_rn(y[0], y[1]); o.x = *reinterpret_cast<uint32_t*>(&t);
        t = __floats2bfloat162_rn(y[2], y[3]); o.y = *reinterpret_cast<uint32_t*>(&t);
        t = __floats2bfloat162_rn(y[4], y[5]); o.z = *reinterpret_cast<uint32_t*>(&t);
        t = __floats2bfloat162_rn(y[6], y[7]); o.w = *reinterpret_cast<uint32_t*>(&t);
        *reinterpret_cast<uint4*>(dst) = o;
      }
    } else {
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(stage + (nl * 128 + ml) * (f32 ? 4 : 2));
    }
  }
}

__device__ __forceinline__ bool epi_needs_rope(int kind) {
  return kind == EPI_QLAT_ROPE || kind == EPI_CACHE_KR || kind == EPI_QP_ROPE;
}
__device__ __forceinline__ double epi_inv_freq(const Epi& e, const TokenMap& tk, int m) {
  if (!epi_needs_rope(e.kind)) return 0.0;
  const int j = (e.kind == EPI_CACHE_KR) ? m : (m % tk.d_R);
  return rope_inv_freq(tk, j >> 1);
}

// (cos, sin) of every rotary pair of the call's T tokens, for the epilogues
// of the GEMMs that follow (one evaluation per (token, pair) instead of one per
// output element).
__global__ void __launch_bounds__(256) rope_table_kernel(const TokenMap tk, int T, float2* out) {
  griddep_wait();  // positions may be written, and the previous call's epilogues may still read `out`
  if (threadIdx.x == 0) griddep_launch_dependents();
  const int half = tk.d_R >> 1;
  const long long total = static_cast<long long>(T) * half;
  for (long long idx = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * 256) {
    const int n = static_cast<int>(idx / half), i = static_cast<int>(idx % half);
    float c, s;
    rope_cos_sin(tok_pos(tk, n), rope_inv_freq(tk, i), c, s);
    out[idx] = make_float2(c, s);
  }
}

}  // namespace mla
