// Decode over the latent cache: query absorption, split-K attention (CUDA-core kernel),
// split merge with W_uv, and the host-side orchestration of one decode step.
//
// Paper notes "MHA2MLA" (ACL 2025), §关键设计: the NoPE key is K_nope = c_kv W_uk and
// the value V = c_kv W_uv (SVDjoint); the RoPE part cannot be merged into the matrices
// and is scored separately.  Absorbing W_uk into the query (q_lat = q_nope W_uk^T)
// scores the NoPE part directly against c_kv; the probability-weighted latent is taken
// through W_uv after the softmax sum.  Scores are kept in log2 units (the query is
// pre-scaled by log2(e)/sqrt(d_h)) so the softmax uses exp2.
#include <algorithm>

#include "decode_common.cuh"

MLA_KSPAN_DEFINE(decode)

namespace mla {

// ------------------------------------------------------------------ absorb_q (+ schedule)
struct AbsorbArgs {
  const void* q;              // [B][H][d_h]
  const int32_t* seq_lens;
  int B, T_cap, H, n_kv, dh, r, d_c, dn, R;
  const void* W_ukT;          // [n_kv][dn][d_c]
  const int32_t* nope_idx;    // [n_kv][dn]
  const int32_t* rope_pair;   // [n_kv][r]
  const double* theta;
  float* qlat;                // f32 [B][H][d_c]        (CUDA-core kernel)
  float* qrope;               // f32 [B][H][2r]
  __nv_bfloat16* qcat;        // bf16 [B][H][K]         (tcgen05 kernel), or null
  int K;
  int bchunk;                 // sequences per CTA
  Sched sched;
  int tile, G;
  int32_t* err;
  int smem_ints;              // dynamic shared memory of the CTA, in ints
  int vec_ok;                 // W_uk rows and q rows allow 16-byte loads
};

constexpr int kAbsRows = 16;   // (b, h) rows per CTA
constexpr int kAbsCols = 64;   // latent columns per CTA

// grid: n_kv * (column chunks) * (row chunks) CTAs, plus one CTA that builds the schedule.
// Each CTA stages its slice of W_uk[g] (all NoPE dims x 64 latent columns) and the NoPE
// query dims of its rows in shared memory, then each thread accumulates 4 rows of one
// latent column.
template <typename T>
__global__ void __launch_bounds__(256) absorb_kernel(AbsorbArgs a) {
  MLA_KSPAN(0);
  const int G = a.H / a.n_kv;
  const int rows_total = a.B * G;
  const int n_rc = (rows_total + kAbsRows - 1) / kAbsRows;
  const int n_cc = (a.d_c + kAbsCols - 1) / kAbsCols;
  if (blockIdx.x == a.n_kv * n_cc * n_rc) {  // the last CTA builds the split-K schedule
    extern __shared__ float sm_sched[];
    build_schedule(a.seq_lens, a.B, a.T_cap, a.tile, a.G, a.sched, a.err, reinterpret_cast<int32_t*>(sm_sched),
                   a.smem_ints);
    return;
  }
  const int g = blockIdx.x % a.n_kv;
  const int cc = (blockIdx.x / a.n_kv) % n_cc;
  const int rc = blockIdx.x / (a.n_kv * n_cc);
  const int row0 = rc * kAbsRows;
  const int rows = min(kAbsRows, rows_total - row0);
  extern __shared__ float sm[];
  float* s_w = sm;                          // [dn][kAbsCols]
  float* s_q = s_w + a.dn * kAbsCols;       // [kAbsRows][dn]
  const float scale = kLog2e * rsqrtf((float)a.dh);
  const T* q = (const T*)a.q;
  const T* W = (const T*)a.W_ukT + (size_t)g * a.dn * a.d_c;
  const int c0 = cc * kAbsCols;
  float* s_qraw = s_q + kAbsRows * a.dn;    // [kAbsRows][dh]
  // all loads of the CTA are issued before any is used (one memory round trip)
  constexpr int VEC = 16 / sizeof(T);
  const bool vec = a.vec_ok && (c0 + kAbsCols <= a.d_c);
  if (vec) {
    constexpr int kMaxW = 8;                 // dn <= 256: dn * 64 / VEC / 256 <= 8 (bf16)
    const int nw = a.dn * (kAbsCols / VEC);
    uint4 wr[kMaxW];
#pragma unroll
    for (int k = 0; k < kMaxW; ++k) {
      const int v = threadIdx.x + 256 * k;
      if (v < nw) {
        const int j = v / (kAbsCols / VEC), part = v % (kAbsCols / VEC);
        wr[k] = __ldg(reinterpret_cast<const uint4*>(W + (size_t)j * a.d_c + c0 + part * VEC));
      }
    }
    const int nq = rows * (a.dh / VEC);
    uint4 qr[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int v = threadIdx.x + 256 * k;
      if (v < nq) {
        const int r = v / (a.dh / VEC), part = v % (a.dh / VEC);
        const int row = row0 + r, b = row / G, h = g * G + row % G;
        qr[k] = __ldg(reinterpret_cast<const uint4*>(q + ((size_t)b * a.H + h) * a.dh + part * VEC));
      }
    }
#pragma unroll
    for (int k = 0; k < kMaxW; ++k) {
      const int v = threadIdx.x + 256 * k;
      if (v < nw) {
        const int j = v / (kAbsCols / VEC), part = v % (kAbsCols / VEC);
        const T* e = reinterpret_cast<const T*>(&wr[k]);
#pragma unroll
        for (int t = 0; t < VEC; ++t) s_w[j * kAbsCols + part * VEC + t] = to_f32(e[t]);
      }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int v = threadIdx.x + 256 * k;
      if (v < nq) {
        const int r = v / (a.dh / VEC), part = v % (a.dh / VEC);
        const T* e = reinterpret_cast<const T*>(&qr[k]);
#pragma unroll
        for (int t = 0; t < VEC; ++t) s_qraw[r * a.dh + part * VEC + t] = to_f32(e[t]);
      }
    }
  } else {
    for (int i = threadIdx.x; i < a.dn * kAbsCols; i += blockDim.x) {
      const int j = i / kAbsCols, cl = i % kAbsCols;
      s_w[i] = (c0 + cl < a.d_c) ? ldg_f32(W + (size_t)j * a.d_c + c0 + cl) : 0.f;
    }
    for (int i = threadIdx.x; i < rows * a.dh; i += blockDim.x) {
      const int r = i / a.dh, e = i % a.dh;
      const int row = row0 + r, b = row / G, h = g * G + row % G;
      s_qraw[i] = ldg_f32(q + ((size_t)b * a.H + h) * a.dh + e);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < rows * a.dn; i += blockDim.x) {
    const int r = i / a.dn, j = i % a.dn;
    s_q[i] = s_qraw[r * a.dh + __ldg(a.nope_idx + g * a.dn + j)];
  }
  if (cc == 0) {
    // RoPE part: rotate the kept pairs at position L-1 (angle in double), scale.
    for (int i = threadIdx.x; i < rows * a.r; i += blockDim.x) {
      const int r = i / a.r, j = i % a.r;
      const int row = row0 + r, b = row / G, h = g * G + row % G;
      const int L = a.seq_lens[b];
      const int p = (L >= 1 && L <= a.T_cap) ? L - 1 : 0;
      const int k = a.rope_pair[g * a.r + j];
      const double x0 = s_qraw[r * a.dh + 2 * k], x1 = s_qraw[r * a.dh + 2 * k + 1];
      double sn, cs;
      sincos((double)p * a.theta[k], &sn, &cs);
      const float o0 = (float)((x0 * cs - x1 * sn) * (double)scale);
      const float o1 = (float)((x0 * sn + x1 * cs) * (double)scale);
      const size_t bh = (size_t)b * a.H + h;
      if (a.qrope) { a.qrope[bh * 2 * a.r + 2 * j] = o0; a.qrope[bh * 2 * a.r + 2 * j + 1] = o1; }
      if (a.qcat && a.K > a.d_c) {
        a.qcat[bh * a.K + a.d_c + g * 2 * a.r + 2 * j] = __float2bfloat16_rn(o0);
        a.qcat[bh * a.K + a.d_c + g * 2 * a.r + 2 * j + 1] = __float2bfloat16_rn(o1);
      }
    }
    if (a.qcat && a.K > a.d_c) {  // zero the other KV heads' RoPE slots of a concatenated row
      for (int i = threadIdx.x; i < rows * a.R; i += blockDim.x) {
        const int r = i / a.R, j = i % a.R;
        if (j / (2 * a.r) == g) continue;
        const int row = row0 + r;
        const size_t bh = (size_t)(row / G) * a.H + g * G + row % G;
        a.qcat[bh * a.K + a.d_c + j] = __float2bfloat16_rn(0.f);
      }
    }
  }
  __syncthreads();
  // q_lat[row][c] = scale * sum_j q_nope[row][j] * W_uk[g][c][j]
  const int cl = threadIdx.x % kAbsCols, rg = threadIdx.x / kAbsCols;  // 4 row groups
  const int c = c0 + cl;
  float acc[kAbsRows / 4];
#pragma unroll
  for (int k = 0; k < kAbsRows / 4; ++k) acc[k] = 0.f;
#pragma unroll 4
  for (int j = 0; j < a.dn; ++j) {
    const float wv = s_w[j * kAbsCols + cl];
#pragma unroll
    for (int k = 0; k < kAbsRows / 4; ++k) acc[k] += s_q[(rg * (kAbsRows / 4) + k) * a.dn + j] * wv;
  }
  if (c < a.d_c) {
#pragma unroll
    for (int k = 0; k < kAbsRows / 4; ++k) {
      const int r = rg * (kAbsRows / 4) + k;
      if (r >= rows) break;
      const int row = row0 + r;
      const size_t bh = (size_t)(row / G) * a.H + g * G + row % G;
      if (a.qlat) a.qlat[bh * a.d_c + c] = acc[k] * scale;
      if (a.qcat) a.qcat[bh * a.K + c] = __float2bfloat16_rn(acc[k] * scale);
    }
  }
}

// ------------------------------------------------------------ CUDA-core split-K decode
struct DecodeArgs {
  mla_cache_t cache;
  int B, H, n_kv, r, d_c, R;
  const float* qlat;
  const float* qrope;
  float* opart;     // [H][P][d_c]
  float* mlpart;    // [H][P][2]
  int P;            // piece capacity
  Sched sched;
};

constexpr int kSimtTile = 32;
constexpr int kSimtMaxE = 32;   // H*d_c / 256 owned accumulators per thread

template <typename T, bool INT4>
__global__ void __launch_bounds__(256) decode_simt_kernel(DecodeArgs a) {
  MLA_KSPAN(1);
  const int H = a.H, dc = a.d_c, R = a.R, r2 = 2 * a.r;
  const int G = H / a.n_kv;
  extern __shared__ float sm[];
  float* s_qlat = sm;                              // [H][dc]
  float* s_qrope = s_qlat + H * dc;                // [H][r2]
  float* s_c = s_qrope + H * r2;                   // [32][dc+1]
  float* s_kr = s_c + kSimtTile * (dc + 1);        // [32][R+1]
  float* s_p = s_kr + kSimtTile * (R + 1);         // [32][H]
  float* s_alpha = s_p + kSimtTile * H;            // [H]
  float* s_m = s_alpha + H;                        // [H]
  float* s_l = s_m + H;                            // [H]
  const int tid = threadIdx.x;
  const int nE = (H * dc + 255) / 256;
  const int w = blockIdx.x;
  for (int pc = a.sched.worker_first[w]; pc < a.sched.worker_first[w + 1]; ++pc) {
    const int b = a.sched.piece_b[pc];
    const int t0 = a.sched.piece_t0[pc], t1 = a.sched.piece_t1[pc];
    for (int i = tid; i < H * dc; i += 256) s_qlat[i] = a.qlat[(size_t)b * H * dc + i];
    for (int i = tid; i < H * r2; i += 256) s_qrope[i] = a.qrope[(size_t)b * H * r2 + i];
    if (tid < H) { s_m[tid] = -INFINITY; s_l[tid] = 0.f; }
    float O[kSimtMaxE];
#pragma unroll
    for (int e = 0; e < kSimtMaxE; ++e) O[e] = 0.f;
    __syncthreads();
    for (int t = t0; t < t1; t += kSimtTile) {
      const int n = min(kSimtTile, t1 - t);
      const size_t slot0 = (size_t)b * a.cache.T_cap + t;
      for (int i = tid; i < n * dc; i += 256) {
        int tt = i / dc, cc = i % dc;
        float v;
        if (INT4) {
          const uint8_t* codes = (const uint8_t*)a.cache.c_kv + (slot0 + tt) * (dc / 2);
          const __half* sc = (const __half*)a.cache.c_scales + (slot0 + tt) * (dc / 32);
          uint32_t byte = codes[cc / 2];
          v = (float)nib_to_int((cc & 1) ? (byte >> 4) : (byte & 15u)) * __half2float(sc[cc / 32]);
        } else {
          v = to_f32(((const T*)a.cache.c_kv)[(slot0 + tt) * dc + cc]);
        }
        s_c[tt * (dc + 1) + cc] = v;
      }
      for (int i = tid; i < n * R; i += 256) {
        int tt = i / R, j = i % R;
        s_kr[tt * (R + 1) + j] =
            to_f32(((const T*)a.cache.k_rope)[mla_kr_offset(b, t + tt, j / r2, j % r2, a.cache.T_cap, a.n_kv, r2)]);
      }
      __syncthreads();
      for (int i = tid; i < n * H; i += 256) {
        int tt = i / H, h = i % H, g = h / G;
        const float* cq = s_qlat + h * dc;
        const float* cc = s_c + tt * (dc + 1);
        float s = 0.f;
        for (int j = 0; j < dc; ++j) s += cq[j] * cc[j];
        const float* rq = s_qrope + h * r2;
        const float* rk = s_kr + tt * (R + 1) + g * r2;
        for (int j = 0; j < r2; ++j) s += rq[j] * rk[j];
        s_p[tt * H + h] = s;
      }
      __syncthreads();
      if (tid < H) {
        float mx = s_m[tid];
        for (int tt = 0; tt < n; ++tt) mx = fmaxf(mx, s_p[tt * H + tid]);
        float al = exp2f(s_m[tid] - mx);   // exp2(-inf) = 0 on the first tile
        float l = s_l[tid] * al;
        for (int tt = 0; tt < n; ++tt) {
          float p = exp2f(s_p[tt * H + tid] - mx);
          s_p[tt * H + tid] = p;
          l += p;
        }
        s_m[tid] = mx; s_l[tid] = l; s_alpha[tid] = al;
      }
      __syncthreads();
#pragma unroll
      for (int e = 0; e < kSimtMaxE; ++e) {
        if (e >= nE) break;
        int idx = tid + 256 * e;
        if (idx < H * dc) {
          int h = idx / dc, cc = idx % dc;
          float acc = O[e] * s_alpha[h];
          for (int tt = 0; tt < n; ++tt) acc += s_p[tt * H + h] * s_c[tt * (dc + 1) + cc];
          O[e] = acc;
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int e = 0; e < kSimtMaxE; ++e) {
      if (e >= nE) break;
      int idx = tid + 256 * e;
      if (idx < H * dc) a.opart[((size_t)(idx / dc) * a.P + pc) * dc + idx % dc] = O[e];
    }
    if (tid < H) {
      a.mlpart[((size_t)tid * a.P + pc) * 2] = s_m[tid];
      a.mlpart[((size_t)tid * a.P + pc) * 2 + 1] = s_l[tid];
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------ combine splits + W_uv
struct CombineArgs {
  int B, H, n_kv, d_c, dh;
  const float* opart;
  const float* mlpart;
  Sched sched;
  const void* W_uv;   // [n_kv][d_c][dh]
  void* out;          // [B][H][dh]
  int bchunk;
  int max_pieces;     // upper bound on pieces per sequence (G + 1)
  int P;              // piece capacity of the partial arrays [H][P]
};

template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  MLA_KSPAN(2);
  const int g = blockIdx.x % a.n_kv, chunk = blockIdx.x / a.n_kv;
  const int G = a.H / a.n_kv;
  const int b0 = chunk * a.bchunk;
  const int nb = min(a.bchunk, a.B - b0);
  const int rows = nb * G;
  extern __shared__ float sm[];
  float* s_o = sm;                      // [rows][d_c] merged latent
  float* s_wt = s_o + rows * a.d_c;     // [rows][max_pieces] merge weights
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  // 1. per (b, h): merge weights 2^(m_j - M) / sum_j 2^(m_j - M) l_j of its pieces
  //    (one warp per row; lanes stride over the pieces)
  for (int row = warp; row < rows; row += nwarp) {
    const int b = b0 + row / G, h = g * G + row % G;
    const int first = a.sched.seq_first[b], np = a.sched.seq_np[b];
    float M = -INFINITY;
    for (int j = lane; j < np; j += 32) M = fmaxf(M, __ldg(a.mlpart + ((size_t)h * a.P + first + j) * 2));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
    for (int j = lane; j < np; j += 32) {
      const float* ml = a.mlpart + ((size_t)h * a.P + first + j) * 2;
      const float wj = exp2f(__ldg(ml) - M);
      s_wt[row * a.max_pieces + j] = wj;
      den += wj * __ldg(ml + 1);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = (np > 0 && den > 0.f) ? 1.f / den : 0.f;
    __syncwarp();
    for (int j = lane; j < np; j += 32) s_wt[row * a.max_pieces + j] *= inv;
  }
  __syncthreads();
  // 2. merged latent: each item is (row, 4 consecutive c); all pieces' loads issued together
  const int c4n = a.d_c / 4;
  for (int it = threadIdx.x; it < rows * c4n; it += blockDim.x) {
    const int row = it / c4n, c4 = it % c4n;
    const int b = b0 + row / G, h = g * G + row % G;
    const int first = a.sched.seq_first[b], np = a.sched.seq_np[b];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < np; j0 += 8) {
      float4 o[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (j0 + k < np)
          o[k] = __ldg(reinterpret_cast<const float4*>(a.opart + ((size_t)h * a.P + first + j0 + k) * a.d_c) + c4);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (j0 + k < np) {
          const float wgt = s_wt[row * a.max_pieces + j0 + k];
          acc.x += wgt * o[k].x; acc.y += wgt * o[k].y; acc.z += wgt * o[k].z; acc.w += wgt * o[k].w;
        }
    }
    *reinterpret_cast<float4*>(&s_o[row * a.d_c + c4 * 4]) = acc;
  }
  __syncthreads();
  // 3. o[row][d] = sum_c O_lat[row][c] W_uv[g][c][d], W_uv[g] staged in chunks of 64 latent
  //    rows (one 16-byte load per thread and chunk row group, all issued before use)
  const T* W = (const T*)a.W_uv + (size_t)g * a.d_c * a.dh;
  float* s_w = s_wt + rows * a.max_pieces;   // [kWc][dh]
  constexpr int kRows = 8, kWc = 64;
  constexpr int VEC = 16 / sizeof(T);
  const int n_items = a.dh * ((rows + kRows - 1) / kRows);
  const int item = threadIdx.x;
  const int d = item % a.dh, r0 = (item / a.dh) * kRows;
  float acc[kRows];
#pragma unroll
  for (int k = 0; k < kRows; ++k) acc[k] = 0.f;
  for (int cb = 0; cb < a.d_c; cb += kWc) {
    const int nc = min(kWc, a.d_c - cb);
    const int nvec = nc * a.dh / VEC;
    uint4 wr[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int v = threadIdx.x + 256 * k;
      if (v < nvec) wr[k] = __ldg(reinterpret_cast<const uint4*>(W + (size_t)cb * a.dh) + v);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int v = threadIdx.x + 256 * k;
      if (v < nvec) {
        const T* e = reinterpret_cast<const T*>(&wr[k]);
#pragma unroll
        for (int t = 0; t < VEC; ++t) s_w[v * VEC + t] = to_f32(e[t]);
      }
    }
    __syncthreads();
    if (item < n_items) {
#pragma unroll 4
      for (int c = 0; c < nc; ++c) {
        const float wv = s_w[c * a.dh + d];
#pragma unroll
        for (int k = 0; k < kRows; ++k)
          if (r0 + k < rows) acc[k] += s_o[(r0 + k) * a.d_c + cb + c] * wv;
      }
    }
    __syncthreads();
  }
  if (item < n_items) {
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
      const int row = r0 + k;
      if (row >= rows) break;
      const int b = b0 + row / G, h = g * G + row % G;
      ((T*)a.out)[((size_t)b * a.H + h) * a.dh + d] = from_f32<T>(acc[k]);
    }
  }
}

template <typename T, bool INT4>
cudaError_t launch_decode_t(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens,
                            const void* q, int B, void* out, void* ws, const DecodeLayout& L,
                            cudaStream_t s) {
  const mla_config_t& cfg = p.cfg;
  const int H = cfg.n_heads, G = H / cfg.n_kv_heads;
  char* base = (char*)ws;
  Sched sched = mla_sched_view(L, ws, B);
  // 1. absorb + schedule
  AbsorbArgs aa;
  aa.q = q; aa.seq_lens = seq_lens; aa.B = B; aa.T_cap = c.T_cap; aa.H = H;
  aa.n_kv = cfg.n_kv_heads; aa.dh = cfg.head_dim; aa.r = cfg.r_pairs; aa.d_c = cfg.d_c;
  aa.dn = p.dn; aa.R = p.R; aa.W_ukT = p.W_ukT; aa.nope_idx = p.nope_idx;
  aa.rope_pair = p.rope_pair; aa.theta = p.theta;
  aa.qlat = L.kernel == 1 ? (float*)(base + L.off_qlat) : nullptr;
  aa.qrope = (float*)(base + L.off_qrope);
  aa.qcat = L.kernel == 2 ? (__nv_bfloat16*)(base + L.off_qlat) : nullptr;
  aa.K = cfg.d_c;
  aa.bchunk = 0;
  aa.sched = sched; aa.tile = L.tile; aa.G = L.G; aa.err = p.err;
  const int n_rc = (B * G + kAbsRows - 1) / kAbsRows, n_cc = (cfg.d_c + kAbsCols - 1) / kAbsCols;
  const size_t smem_abs = std::max((size_t)(p.dn * kAbsCols + kAbsRows * p.dn + kAbsRows * cfg.head_dim) * sizeof(float),
                                    (size_t)(4 * B + 1) * sizeof(int32_t));
  {
    const int vecn = 16 / (int)sizeof(T);  // elements per 16-byte load
    aa.vec_ok = ((uintptr_t)q % 16 == 0) && cfg.d_c % vecn == 0 && cfg.head_dim % vecn == 0 &&
                p.dn * (kAbsCols / vecn) <= 256 * 8 && kAbsRows * (cfg.head_dim / vecn) <= 256 * 2;
  }
  aa.smem_ints = (int)(smem_abs / sizeof(int32_t));
  cudaError_t e = cudaFuncSetAttribute(absorb_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_abs);
  if (e != cudaSuccess) return e;
  absorb_kernel<T><<<cfg.n_kv_heads * n_cc * n_rc + 1, 256, smem_abs, s>>>(aa);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 2. split-K attention over the latent cache
  if (L.kernel == 1) {
    DecodeArgs da;
    da.cache = c; da.B = B; da.H = H; da.n_kv = cfg.n_kv_heads; da.r = cfg.r_pairs;
    da.d_c = cfg.d_c; da.R = p.R; da.qlat = aa.qlat; da.qrope = aa.qrope;
    da.opart = (float*)(base + L.off_opart); da.mlpart = (float*)(base + L.off_mlpart);
    da.P = L.P;
    da.sched = sched;
    size_t smem = sizeof(float) * ((size_t)H * cfg.d_c + H * 2 * cfg.r_pairs +
                                   kSimtTile * (cfg.d_c + 1) + kSimtTile * (p.R + 1) +
                                   kSimtTile * H + 3 * H);
    e = cudaFuncSetAttribute(decode_simt_kernel<T, INT4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    if ((e = mla_profile_event(p, 0, s)) != cudaSuccess) return e;
    decode_simt_kernel<T, INT4><<<L.G, 256, smem, s>>>(da);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if ((e = mla_profile_event(p, 1, s)) != cudaSuccess) return e;
  } else {
    e = mla_launch_decode_tc(p, c, B, sched, base + L.off_qlat, (const float*)(base + L.off_qrope),
                             (float*)(base + L.off_opart), (float*)(base + L.off_mlpart), L.P, L.G, s);
    if (e != cudaSuccess) return e;
  }
  // 3. merge the splits and apply W_uv
  CombineArgs ca;
  ca.B = B; ca.H = H; ca.n_kv = cfg.n_kv_heads; ca.d_c = cfg.d_c; ca.dh = cfg.head_dim;
  ca.opart = (const float*)(base + L.off_opart); ca.mlpart = (const float*)(base + L.off_mlpart);
  ca.sched = sched; ca.W_uv = p.W_uv; ca.out = out; ca.P = L.P;
  // rows (b, h) per CTA: at most 8 per thread and 256 / d_h row groups
  const int rows_cta = std::max(G, (8 * std::max(1, 256 / cfg.head_dim)) / G * G);
  ca.bchunk = std::max(1, rows_cta / G);
  const int cchunks = (B + ca.bchunk - 1) / ca.bchunk;
  ca.max_pieces = L.G + 1;
  const size_t smem_c =
      ((size_t)ca.bchunk * G * (cfg.d_c + ca.max_pieces) + 64 * (size_t)cfg.head_dim) * sizeof(float);
  e = cudaFuncSetAttribute(combine_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_c);
  if (e != cudaSuccess) return e;
  combine_kernel<T><<<cfg.n_kv_heads * cchunks, 256, smem_c, s>>>(ca);
  return cudaGetLastError();
}

}  // namespace mla

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

DecodeLayout mla_decode_layout(const mla_plan& p, int B, int kernel) {
  const mla_config_t& cfg = p.cfg;
  DecodeLayout L;
  L.kernel = kernel;
  L.tile = kernel == 2 ? 128 : mla::kSimtTile;
  L.G = p.opt_splits > 0 ? p.opt_splits : (kernel == 2 ? p.num_sms : 2 * p.num_sms);
  L.P = B + L.G;
  L.K = cfg.d_c + p.R;
  const int H = cfg.n_heads;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align256(o + bytes); return r; };
  L.off_seq_tile0 = take(sizeof(int32_t) * B);
  L.off_seq_ntiles = take(sizeof(int32_t) * B);
  L.off_seq_ne = take(sizeof(int32_t) * (B + 1));
  L.off_seq_first = take(sizeof(int32_t) * B);
  L.off_seq_np = take(sizeof(int32_t) * B);
  L.off_worker_first = take(sizeof(int32_t) * (L.G + 1));
  L.off_piece_b = take(sizeof(int32_t) * L.P);
  L.off_piece_t0 = take(sizeof(int32_t) * L.P);
  L.off_piece_t1 = take(sizeof(int32_t) * L.P);
  if (L.kernel == 1)
    L.off_qlat = take(sizeof(float) * (size_t)B * H * cfg.d_c);          // f32 absorbed query
  else
    L.off_qlat = take(sizeof(uint16_t) * (size_t)B * H * cfg.d_c);       // bf16 absorbed query
  L.off_qrope = take(sizeof(float) * (size_t)B * H * 2 * cfg.r_pairs + 4);
  L.off_opart = take(sizeof(float) * (size_t)L.P * H * cfg.d_c);
  L.off_mlpart = take(sizeof(float) * (size_t)L.P * H * 2);
  L.total = o;
  return L;
}

Sched mla_sched_view(const DecodeLayout& L, void* ws, int B) {
  char* b = (char*)ws;
  Sched s;
  s.seq_tile0 = (int32_t*)(b + L.off_seq_tile0);
  s.seq_ntiles = (int32_t*)(b + L.off_seq_ntiles);
  s.seq_ne = (int32_t*)(b + L.off_seq_ne);
  s.seq_first = (int32_t*)(b + L.off_seq_first);
  s.seq_np = (int32_t*)(b + L.off_seq_np);
  s.worker_first = (int32_t*)(b + L.off_worker_first);
  s.piece_b = (int32_t*)(b + L.off_piece_b);
  s.piece_t0 = (int32_t*)(b + L.off_piece_t0);
  s.piece_t1 = (int32_t*)(b + L.off_piece_t1);
  return s;
}

cudaError_t mla_launch_decode(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens,
                              const void* q, int B, void* out, void* ws, const DecodeLayout& L,
                              cudaStream_t s) {
  using namespace mla;
  bool int4 = p.cfg.cache_kind == MLA_CACHE_INT4_G32;
  if (p.cfg.dtype == MLA_BF16)
    return int4 ? launch_decode_t<__nv_bfloat16, true>(p, c, seq_lens, q, B, out, ws, L, s)
                : launch_decode_t<__nv_bfloat16, false>(p, c, seq_lens, q, B, out, ws, L, s);
  return launch_decode_t<float, false>(p, c, seq_lens, q, B, out, ws, L, s);
}
