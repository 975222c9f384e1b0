// Decode over the latent cache: query absorption, split-K attention (CUDA-core kernel),
// split merge with W_uv, and the host-side orchestration of one decode step.
//
// Paper notes "MHA2MLA" (ACL 2025), §关键设计: the NoPE key is K_nope = c_kv W_uk and
// the value V = c_kv W_uv (SVDjoint); the RoPE part cannot be merged into the matrices
// and is scored separately.  Absorbing W_uk into the query (q_lat = q_nope W_uk^T)
// scores the NoPE part directly against c_kv; the probability-weighted latent is taken
// through W_uv after the softmax sum.  Scores are kept in log2 units (the query is
// pre-scaled by log2(e)/sqrt(d_h)) so the softmax uses exp2.
#include <math.h>

#include <algorithm>

#include "append_common.cuh"
#include "decode_common.cuh"

#include <type_traits>


namespace mla {

// ------------------------------------------------------------------ absorb_q (+ schedule)
struct AbsorbArgs {
  const void* q;              // [B][H][d_h]
  const int32_t* seq_lens;
  int B, T_cap, H, n_kv, dh, r, d_c;
  const void* W_ukF;          // [n_kv][d_h][d_c]: W_uk^T on the NoPE dims, zero rows on the kept pairs
  const int32_t* rope_pair;   // [n_kv][r]
  const double* theta;
  float* qlat;                // f32 [B][H][d_c]        (CUDA-core kernel), or null
  __nv_bfloat16* qlat16;      // bf16 [B][H][d_c]       (tcgen05 kernels), or null
  float* qrope;               // f32 [B][H][2r]
  Sched sched;
  int tile, G;
  int32_t* err;
  int sched_ints;             // shared memory of the schedule CTA, in ints
  float sm_scale;             // softmax scale of the scores (1/sqrt(d_h) unless the config sets one)
  int vec_ok;                 // q and W rows allow 16-byte loads
  int mma;                    // product as bf16 warp MMAs (32 rows per CTA), else CUDA cores (8 rows)
  // many queries per sequence: query rows s = b * q_chunk + i sit at position
  // seq_lens[b] - q_chunk + i; the schedule runs over units of q_block queries (1, 1: decode)
  int q_chunk, q_block;
};

constexpr int kAbsRows = 8;       // (b, h) rows per CTA, CUDA-core form: one per warp
constexpr int kAbsRowsMma = 32;   // rows per CTA, warp-MMA form: two m16 tiles
constexpr int kAbsCols = 64;      // latent columns per CTA

// Block `blk` of the absorption grid: block 0 builds the split-K schedule (dispatched
// first), blocks 1 .. n_kv * (row blocks) * (column chunks) compute
//     q_lat[row][c] = scale * sum_d q[row][d] * W_ukF[g][d][c]
// for a block of (b, h) rows of KV head g and 64 latent columns.  W_ukF carries W_uk^T on
// the NoPE dims and zero rows on the kept pairs' dims, so the unrotated query is used as it
// is (no NoPE gather).  The kept pairs of the first column chunk's rows are rotated at the
// query's position (angle in double) and scaled into q_rope.  What comes from the plan
// (W_ukF slice, pair table, frequencies) is staged before the dependency wait, the
// caller's queries and lengths after it.  `sm` is the CTA's dynamic shared memory.
template <typename T>
__device__ __forceinline__ void absorb_body(const AbsorbArgs& a, int blk_id, float* sm) {
  const int G = a.H / a.n_kv;
  const int rows_total = a.B * G;
  const int RPC = a.mma ? kAbsRowsMma : kAbsRows;
  const int n_rb = (rows_total + RPC - 1) / RPC;
  if (blk_id == 0) {  // the split-K schedule
    const int nunits = a.q_chunk > 1 ? (a.B / a.q_chunk) * ((a.q_chunk + a.q_block - 1) / a.q_block) : a.B;
    build_schedule(a.seq_lens, nunits, a.T_cap, a.tile, a.G, a.sched, a.err, reinterpret_cast<int32_t*>(sm),
                   a.sched_ints, a.q_chunk, a.q_block);
    return;
  }
  const int blk = blk_id - 1;
  const int g = blk % a.n_kv;
  const int rb = (blk / a.n_kv) % n_rb;
  const int cc = blk / (a.n_kv * n_rb);
  const int row0 = rb * RPC, c0 = cc * kAbsCols;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int dh = a.dh;
  const T* q = (const T*)a.q;
  const T* W = (const T*)a.W_ukF + (size_t)g * dh * a.d_c;
  const float scale = kLog2e * a.sm_scale;
  const int nrow = min(RPC, rows_total - row0);
  auto q_row = [&](int r) {   // query row r of this CTA
    const int row = row0 + r;
    return q + ((size_t)(row / G) * a.H + g * G + row % G) * dh;
  };
  auto out_index = [&](int row, int c) { return ((size_t)(row / G) * a.H + g * G + row % G) * a.d_c + c; };
  // RoPE query part (first column chunk): rotate the kept pairs at the query's position
  // (angle in double), scale.  qv(r, d) reads element d of staged row r.
  auto rope = [&](auto qv) {
    if (cc != 0) return;
    for (int item = tid; item < nrow * a.r; item += blockDim.x) {
      const int r = item / a.r, jr = item % a.r, row = row0 + r;
      const int k = __ldg(a.rope_pair + g * a.r + jr);
      const int sq = row / G;
      const int L = __ldg(a.seq_lens + sq / a.q_chunk) - (a.q_chunk - 1 - sq % a.q_chunk);
      const int p = (L >= 1 && L <= a.T_cap) ? L - 1 : 0;
      const double x0 = qv(r, 2 * k), x1 = qv(r, 2 * k + 1);
      float sn, cs;
      rope_sincos(p, __ldg(a.theta + k), &sn, &cs);
      const size_t o = ((size_t)sq * a.H + g * G + row % G) * 2 * a.r + 2 * jr;
      a.qrope[o] = (float)((x0 * cs - x1 * sn) * (double)scale);
      a.qrope[o + 1] = (float)((x0 * sn + x1 * cs) * (double)scale);
    }
  };

  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (a.mma) {
      // ---- warp-MMA form: Qs [32][KP+8] and Ws [KP][64+8] bf16 tiles (16-byte padded rows,
      // conflict-free ldmatrix), staged with 16-byte asynchronous copies (zero-filled past
      // the matrix edges); warps 0-3 each take 16 columns x 32 rows, K = d_h
      using bf16 = __nv_bfloat16;
      const int KP = (dh + 15) & ~15, QLD = KP + 8;
      constexpr int WLD = kAbsCols + 8;
      bf16* Ws = reinterpret_cast<bf16*>(sm);   // [KP][WLD]
      bf16* Qs = Ws + KP * WLD;                 // [32][QLD]
      for (int v = tid; v < KP * (kAbsCols / 8); v += blockDim.x) {
        const int d = v / (kAbsCols / 8), part = v % (kAbsCols / 8), c = c0 + part * 8;
        const bool ok = d < dh && c + 8 <= a.d_c;
        sm100::cp_async16(wmma16::smem_addr(Ws + d * WLD + part * 8),
                          ok ? (const void*)(W + (size_t)d * a.d_c + c) : a.W_ukF, ok ? 16u : 0u);
      }
      sm100::cp_async_commit();
      pdl_wait();
      pdl_trigger();
      for (int v = tid; v < kAbsRowsMma * (KP / 8); v += blockDim.x) {
        const int r = v / (KP / 8), ch = v % (KP / 8);
        const bool ok = r < nrow && ch * 8 + 8 <= dh;
        sm100::cp_async16(wmma16::smem_addr(Qs + r * QLD + ch * 8), ok ? (const void*)(q_row(r) + ch * 8) : a.q,
                          ok ? 16u : 0u);
      }
      sm100::cp_async_commit();
      sm100::cp_async_wait_all();
      __syncthreads();
      rope([&](int r, int d) { return (double)__bfloat162float(Qs[r * QLD + d]); });
      if (warp < 4) {
        float acc[2][2][4] = {};
        for (int k0 = 0; k0 < KP; k0 += 16) {
          uint32_t af[2][4], bfr[4];
          wmma16::load_a(af[0], Qs, QLD, 0, k0, lane);
          wmma16::load_a(af[1], Qs, QLD, 16, k0, lane);
          wmma16::load_b2(bfr, Ws, WLD, k0, 16 * warp, lane);
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            wmma16::mma_16816(acc[m][0], af[m], bfr[0], bfr[1]);
            wmma16::mma_16816(acc[m][1], af[m], bfr[2], bfr[3]);
          }
        }
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
              const int r = 16 * m + (lane >> 2) + 8 * hlf, c = c0 + 16 * warp + 8 * nt + 2 * (lane & 3);
              if (r >= nrow || c >= a.d_c) continue;
              const float v0 = acc[m][nt][2 * hlf] * scale, v1 = acc[m][nt][2 * hlf + 1] * scale;
              const size_t o = out_index(row0 + r, c);
              if (a.qlat16) *reinterpret_cast<__nv_bfloat162*>(a.qlat16 + o) = __floats2bfloat162_rn(v0, v1);
              if (a.qlat) *reinterpret_cast<float2*>(a.qlat + o) = make_float2(v0, v1);
            }
      }
      return;
    }
  }
  // ---- CUDA-core form: W slice and query rows as float in shared memory; warp r takes
  // row r, lane l columns 2l, 2l+1 of the chunk
  float* s_w = sm;                              // [dh][kAbsCols]
  float* s_q = s_w + dh * kAbsCols;             // [kAbsRows][dh]
  const int ncol = min(kAbsCols, a.d_c - c0);
  if (ncol < kAbsCols)
    for (int i = tid; i < dh * kAbsCols; i += blockDim.x) s_w[i] = 0.f;   // columns past d_c
  stage_rows_f32<T>(s_w, kAbsCols, dh, ncol, a.vec_ok && ncol == kAbsCols,
                    [&](int j) { return W + (size_t)j * a.d_c + c0; });
  pdl_wait();
  pdl_trigger();
  stage_rows_f32<T>(s_q, dh, nrow, dh, a.vec_ok, q_row);
  __syncthreads();
  rope([&](int r, int d) { return (double)s_q[r * dh + d]; });
  const int r = warp, row = row0 + r, c = c0 + 2 * lane;
  const float* qn = s_q + r * dh;
  float acc0 = 0.f, acc1 = 0.f;
  int j = 0;
  for (; j + 4 <= dh; j += 4) {
    const float4 x = *reinterpret_cast<const float4*>(qn + j);
    const float2 w0 = *reinterpret_cast<const float2*>(s_w + (j + 0) * kAbsCols + 2 * lane);
    const float2 w1 = *reinterpret_cast<const float2*>(s_w + (j + 1) * kAbsCols + 2 * lane);
    const float2 w2 = *reinterpret_cast<const float2*>(s_w + (j + 2) * kAbsCols + 2 * lane);
    const float2 w3 = *reinterpret_cast<const float2*>(s_w + (j + 3) * kAbsCols + 2 * lane);
    acc0 += x.x * w0.x + x.y * w1.x + x.z * w2.x + x.w * w3.x;
    acc1 += x.x * w0.y + x.y * w1.y + x.z * w2.y + x.w * w3.y;
  }
  for (; j < dh; ++j) {
    const float2 w = *reinterpret_cast<const float2*>(s_w + j * kAbsCols + 2 * lane);
    acc0 += qn[j] * w.x;
    acc1 += qn[j] * w.y;
  }
  if (r < nrow && c < a.d_c) {
    const size_t o = out_index(row, c);
    if (a.qlat) {
      a.qlat[o] = acc0 * scale;
      if (c + 1 < a.d_c) a.qlat[o + 1] = acc1 * scale;
    }
    if (a.qlat16) {
      a.qlat16[o] = __float2bfloat16_rn(acc0 * scale);
      if (c + 1 < a.d_c) a.qlat16[o + 1] = __float2bfloat16_rn(acc1 * scale);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) absorb_kernel(AbsorbArgs a) {
  extern __shared__ __align__(16) float sm[];
  absorb_body<T>(a, blockIdx.x, sm);
}

// ------------------------------------------------------------ CUDA-core split-K decode
struct DecodeArgs {
  mla_cache_t cache;
  const int32_t* seq_lens;   // read for the residual window only
  int32_t* err;
  int qbits;                 // quantised cache: code width (4 or 2)
  int B, H, n_kv, r, d_c, R;
  const float* qlat;
  const float* qrope;
  float* opart;     // [P][H][d_c]
  float* mlpart;    // [H][P][2]
  int P;            // piece capacity
  Sched sched;
};

constexpr int kSimtTile = 32;
constexpr int kSimtMaxE = 32;   // H*d_c / 256 owned accumulators per thread

template <typename T, bool INT4>
__global__ void __launch_bounds__(256) decode_simt_kernel(DecodeArgs a) {
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
  pdl_wait();   // schedule and absorbed queries
  pdl_trigger();
  for (int pc = a.sched.worker_first[w]; pc < a.sched.worker_first[w + 1]; ++pc) {
    const int b = a.sched.piece_b[pc];
    const int t0 = a.sched.piece_t0[pc], t1 = a.sched.piece_t1[pc];
    for (int i = tid; i < H * dc; i += 256) s_qlat[i] = a.qlat[(size_t)b * H * dc + i];
    for (int i = tid; i < H * r2; i += 256) s_qrope[i] = a.qrope[(size_t)b * H * r2 + i];
    if (tid < H) { s_m[tid] = -INFINITY; s_l[tid] = 0.f; }
    // residual window: tokens from lo on may be read unquantised from the ring
    const int lo = (INT4 && a.cache.c_resid) ? __ldg(a.seq_lens + b) - MLA_RESID_WINDOW : INT_MAX;
    float O[kSimtMaxE];
#pragma unroll
    for (int e = 0; e < kSimtMaxE; ++e) O[e] = 0.f;
    __syncthreads();
    for (int t = t0; t < t1; t += kSimtTile) {
      const int n = min(kSimtTile, t1 - t);
      const MlaLoc lc = mla_loc(a.cache, b, t, a.err);   // a 32-token tile lies in one block
      const size_t slot0 = (size_t)lc.pb * lc.cap + lc.pt;
      for (int i = tid; i < n * dc; i += 256) {
        int tt = i / dc, cc = i % dc;
        float v;
        if (INT4) {
          const int tp = t + tt;
          const size_t rs = (size_t)b * MLA_RESID_WINDOW + (tp & (MLA_RESID_WINDOW - 1));
          if (tp >= lo && a.cache.resid_pos[rs] == tp) {
            v = __bfloat162float(((const __nv_bfloat16*)a.cache.c_resid)[rs * dc + cc]);
          } else if (a.qbits == 4) {
            const uint8_t* codes = (const uint8_t*)a.cache.c_kv + (slot0 + tt) * (dc / 2);
            const __half* sc = (const __half*)a.cache.c_scales + (slot0 + tt) * (dc / 32);
            uint32_t byte = codes[cc / 2];
            v = (float)nib_to_int((cc & 1) ? (byte >> 4) : (byte & 15u)) * __half2float(sc[cc / 32]);
          } else {   // 2-bit: element 4i+k in bits 2k..2k+1 of byte i, two's complement
            const uint8_t* codes = (const uint8_t*)a.cache.c_kv + (slot0 + tt) * (dc / 4);
            const __half* sc = (const __half*)a.cache.c_scales + (slot0 + tt) * (dc / 32);
            const int f = (codes[cc / 4] >> (2 * (cc & 3))) & 3;
            v = (float)(f >= 2 ? f - 4 : f) * __half2float(sc[cc / 32]);
          }
        } else {
          v = to_f32(((const T*)a.cache.c_kv)[(slot0 + tt) * dc + cc]);
        }
        s_c[tt * (dc + 1) + cc] = v;
      }
      for (int i = tid; i < n * R; i += 256) {
        int tt = i / R, j = i % R;
        s_kr[tt * (R + 1) + j] =
            to_f32(((const T*)a.cache.k_rope)[mla_kr_offset(lc.pb, lc.pt + tt, j / r2, j % r2, lc.cap, a.n_kv, r2)]);
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
      if (idx < H * dc) a.opart[((size_t)pc * H + idx / dc) * dc + idx % dc] = O[e];
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
  int P;              // piece capacity of the partial arrays [H][P]
  int ncols;          // output columns per CTA: 64, or 32 when the latent is wide
  int vec_ok;         // W_uv rows allow 16-byte loads
  // Many queries per sequence: the merged units are (sequence, block of q_block queries)
  // with H = q_block * heads rows each; row h of unit v is query (v % nqb) * q_block +
  // h / heads of sequence v / nqb, head h % heads (W_uv group (h % heads) / G).  Decode:
  // q_chunk = q_block = 1, heads = H.
  int q_chunk, q_block, heads;
  int rpw;            // rows per warp: a CTA merges 8 rpw rows against one staged W_uv chunk
};

// Output row (query row x head) of merged row h of unit v, or -1 past the chunk's last query.
__device__ __forceinline__ long long combine_out_row(const CombineArgs& a, int v, int h) {
  if (a.q_chunk <= 1) return (long long)v * a.H + h;
  const int nqb = (a.q_chunk + a.q_block - 1) / a.q_block;
  const int i = (v % nqb) * a.q_block + h / a.heads;
  if (i >= a.q_chunk) return -1;
  return ((long long)(v / nqb) * a.q_chunk + i) * a.heads + h % a.heads;
}

constexpr int kCmbRows = 8;    // warps per CTA; a warp merges rpw rows (b, h)
constexpr int kCmbMaxRpw = 4;

// grid: n_kv * (row blocks of 8 rpw rows) * (output column chunks).  Before the dependency
// wait the CTA stages its W_uv[g] column chunk; after it, warp r merges the pieces of rows
// r, r + 8, ... of its block,
//     O_lat = sum_j 2^(m_j - M) O_j / sum_j 2^(m_j - M) l_j,
// into shared memory (all of a batch of pieces' loads in flight together), and then
// out[row][d] = sum_c O_lat[row][c] W_uv[g][c][d] with lane l on columns 2l, 2l+1.
template <typename T>
__global__ void __launch_bounds__(256, 2) combine_kernel(CombineArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int G = a.H / a.n_kv;
  const int rows_total = a.B * G;
  const int RB = kCmbRows * a.rpw;            // rows of this CTA
  const int RBP = (RB + 15) & ~15;            // padded to whole m16 tiles
  const int n_rb = (rows_total + RB - 1) / RB;
  const int g = blockIdx.x % a.n_kv;
  const int rb = (blockIdx.x / a.n_kv) % n_rb;
  const int dcb = blockIdx.x / (a.n_kv * n_rb);
  const int NCOL = a.ncols;
  const int row0 = rb * RB, d0 = dcb * NCOL;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int dc = a.d_c;
  // bf16 with whole 16-byte rows: the output product runs as warp MMAs on bf16 tiles
  const bool mma = std::is_same<T, __nv_bfloat16>::value && a.vec_ok && NCOL == 64 && d0 + 64 <= a.dh;
  constexpr int WLD = 64 + 8;            // bf16 W tile row stride (conflict-free ldmatrix)
  const int ALD = dc + 8;                // bf16 A tile row stride
  float* s_w = sm;                       // f32 [d_c][NCOL], or bf16 [d_c][WLD] for the MMA form
  float* s_o = s_w + dc * NCOL;          // [RB][d_c]
  __nv_bfloat16* s_a = reinterpret_cast<__nv_bfloat16*>(s_o + RB * dc);   // [RBP][ALD]
  const T* W = (const T*)a.W_uv + (size_t)(g % (a.heads / G)) * dc * a.dh;
  const int ncol = min(NCOL, a.dh - d0);
  if (mma) {
    __nv_bfloat16* wt = reinterpret_cast<__nv_bfloat16*>(s_w);
    for (int v = tid; v < dc * 8; v += 256) {
      const int c = v >> 3, part = v & 7;
      sm100::cp_async16(wmma16::smem_addr(wt + c * WLD + part * 8), W + (size_t)c * a.dh + d0 + part * 8, 16u);
    }
    sm100::cp_async_commit();
  } else {
    if (ncol < NCOL)
      for (int i = tid; i < dc * NCOL; i += 256) s_w[i] = 0.f;   // columns past d_h
    stage_rows_f32<T>(s_w, NCOL, dc, ncol, a.vec_ok && ncol == NCOL, [&](int c) { return W + (size_t)c * a.dh + d0; });
  }
  // the schedule was written two kernels back (complete before the attention kernel let
  // this one launch); the partials need the dependency wait
  int firsts[kCmbMaxRpw], nps[kCmbMaxRpw];
#pragma unroll
  for (int j = 0; j < kCmbMaxRpw; ++j) {
    firsts[j] = 0;
    nps[j] = 0;
    const int row = row0 + warp + kCmbRows * j;
    if (j < a.rpw && row < rows_total) {
      const int b = row / G;
      firsts[j] = __ldg(a.sched.seq_first + b);
      nps[j] = __ldg(a.sched.seq_np + b);
    }
  }
  pdl_wait();   // the partials of the attention kernel
  pdl_trigger();
#pragma unroll 1
  for (int j = 0; j < a.rpw; ++j) {
    int first = firsts[0], np = nps[0];
#pragma unroll
    for (int k = 1; k < kCmbMaxRpw; ++k)
      if (j == k) { first = firsts[k]; np = nps[k]; }
    const int r = warp + kCmbRows * j, row = row0 + r;
    float* o = s_o + r * dc;
    if (row < rows_total) {
      const int h = g * G + row % G;
      const float* ml = a.mlpart + ((size_t)h * a.P + first) * 2;
      const float* op = a.opart + ((size_t)first * a.H + h) * dc;   // piece j at op + j * H * d_c
      const size_t ps = (size_t)a.H * dc;
      // pieces j = lane (+32k): running max and sum; the first 8 pieces' latent rows are
      // loaded in the same round trip (they do not depend on the weights)
      const int nc4 = dc / 4;
      float4 v0[8], v1[8];   // columns lane and lane + 32 (float4 units) of pieces 0..7
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (k < np) {
          if (lane < nc4) v0[k] = __ldg(reinterpret_cast<const float4*>(op + (size_t)k * ps) + lane);
          if (lane + 32 < nc4) v1[k] = __ldg(reinterpret_cast<const float4*>(op + (size_t)k * ps) + lane + 32);
        }
      }
      float mj = -INFINITY, lj = 0.f;
      if (lane < np) { mj = __ldg(ml + 2 * lane); lj = __ldg(ml + 2 * lane + 1); }
      float M = mj;
      for (int j = lane + 32; j < np; j += 32) M = fmaxf(M, __ldg(ml + 2 * j));
#pragma unroll
      for (int s = 16; s > 0; s >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, s));
      const float wl = lane < np ? exp2f(mj - M) : 0.f;   // weight of piece `lane`
      float den = wl * lj;
      for (int j = lane + 32; j < np; j += 32) den += exp2f(__ldg(ml + 2 * j) - M) * __ldg(ml + 2 * j + 1);
#pragma unroll
      for (int s = 16; s > 0; s >>= 1) den += __shfl_xor_sync(0xffffffffu, den, s);
      const float inv = (np > 0 && den > 0.f) ? 1.f / den : 0.f;
      float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (k < np) {
          const float w = __shfl_sync(0xffffffffu, wl, k);
          a0.x += w * v0[k].x; a0.y += w * v0[k].y; a0.z += w * v0[k].z; a0.w += w * v0[k].w;
          a1.x += w * v1[k].x; a1.y += w * v1[k].y; a1.z += w * v1[k].z; a1.w += w * v1[k].w;
        }
      }
      for (int j = 8; j < np; ++j) {   // more than 8 pieces: one at a time
        const float w = j < 32 ? __shfl_sync(0xffffffffu, wl, j) : exp2f(__ldg(ml + 2 * j) - M);
        if (lane < nc4) {
          const float4 x = __ldg(reinterpret_cast<const float4*>(op + (size_t)j * ps) + lane);
          a0.x += w * x.x; a0.y += w * x.y; a0.z += w * x.z; a0.w += w * x.w;
        }
        if (lane + 32 < nc4) {
          const float4 x = __ldg(reinterpret_cast<const float4*>(op + (size_t)j * ps) + lane + 32);
          a1.x += w * x.x; a1.y += w * x.y; a1.z += w * x.z; a1.w += w * x.w;
        }
      }
      if (lane < nc4) *reinterpret_cast<float4*>(o + 4 * lane) = make_float4(a0.x * inv, a0.y * inv, a0.z * inv, a0.w * inv);
      if (lane + 32 < nc4)
        *reinterpret_cast<float4*>(o + 4 * lane + 128) = make_float4(a1.x * inv, a1.y * inv, a1.z * inv, a1.w * inv);
      for (int c4 = lane + 64; c4 < nc4; c4 += 32) {   // latents wider than 256
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < np; ++j) {
          const float w = j < 32 ? __shfl_sync(0xffffffffu, wl, j) : exp2f(__ldg(ml + 2 * j) - M);
          const float4 x = __ldg(reinterpret_cast<const float4*>(op + (size_t)j * ps) + c4);
          acc.x += w * x.x; acc.y += w * x.y; acc.z += w * x.z; acc.w += w * x.w;
        }
        *reinterpret_cast<float4*>(o + 4 * c4) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      }
    } else {
      for (int c = lane; c < dc; c += 32) o[c] = 0.f;
    }
  }
  if (mma) {
    // A = merged rows as bf16 (pad rows zero), B = W_uv chunk: 16-row tiles x 16-column
    // slices, one (tile, slice) pair per warp at a time
    __syncthreads();   // every warp's merged rows are in s_o
    for (int i = tid; i < RBP * dc; i += 256) {
      const int r = i / dc, c = i % dc;
      s_a[r * ALD + c] = __float2bfloat16_rn(r < RB ? s_o[r * dc + c] : 0.f);
    }
    sm100::cp_async_wait_all();
    __syncthreads();
    const __nv_bfloat16* wt = reinterpret_cast<const __nv_bfloat16*>(s_w);
    for (int job = warp; job < (RBP / 16) * 4; job += kCmbRows) {
      const int mt = job >> 2, ns = job & 3;   // row tile, 16-column slice
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      for (int k0 = 0; k0 < dc; k0 += 16) {
        uint32_t af[4], bf[4];
        wmma16::load_a(af, s_a, ALD, 16 * mt, k0, lane);
        wmma16::load_b2(bf, wt, WLD, k0, 16 * ns, lane);
        wmma16::mma_16816(acc[0], af, bf[0], bf[1]);
        wmma16::mma_16816(acc[1], af, bf[2], bf[3]);
      }
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {   // fragment rows lane / 4 and lane / 4 + 8
        const int r = 16 * mt + (lane >> 2) + 8 * hr, row = row0 + r;
        const long long orow = r < RB && row < rows_total ? combine_out_row(a, row / G, g * G + row % G) : -1;
        if (orow < 0) continue;
        T* out = (T*)a.out + (size_t)orow * a.dh + d0 + 16 * ns + 2 * (lane & 3);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          __nv_bfloat162 v = __floats2bfloat162_rn(acc[j][2 * hr], acc[j][2 * hr + 1]);
          *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(out) + 8 * j) = v;
        }
      }
    }
    return;
  }
  __syncthreads();
  const int d = d0 + 2 * lane;
  if (2 * lane >= NCOL) return;
  for (int j = 0; j < a.rpw; ++j) {
  const int r = warp + kCmbRows * j, row = row0 + r;
  const float* o = s_o + r * dc;
  float acc0 = 0.f, acc1 = 0.f;
  for (int c = 0; c < dc; c += 4) {
    const float4 x = *reinterpret_cast<const float4*>(o + c);
    const float2 w0 = *reinterpret_cast<const float2*>(s_w + (c + 0) * NCOL + 2 * lane);
    const float2 w1 = *reinterpret_cast<const float2*>(s_w + (c + 1) * NCOL + 2 * lane);
    const float2 w2 = *reinterpret_cast<const float2*>(s_w + (c + 2) * NCOL + 2 * lane);
    const float2 w3 = *reinterpret_cast<const float2*>(s_w + (c + 3) * NCOL + 2 * lane);
    acc0 += x.x * w0.x + x.y * w1.x + x.z * w2.x + x.w * w3.x;
    acc1 += x.x * w0.y + x.y * w1.y + x.z * w2.y + x.w * w3.y;
  }
  const long long orow = row < rows_total ? combine_out_row(a, row / G, g * G + row % G) : -1;
  if (orow >= 0 && d < a.dh) {
    T* out = (T*)a.out + (size_t)orow * a.dh + d;
    out[0] = from_f32<T>(acc0);
    if (d + 1 < a.dh) out[1] = from_f32<T>(acc1);
  }
  }
}

// Arguments and shared memory of the absorption grid (block 0: the split-K schedule).
template <typename T>
void absorb_setup(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, const void* q, int B, void* ws,
                  const DecodeLayout& L, AbsorbArgs* aa, size_t* smem, int* nblocks) {
  const mla_config_t& cfg = p.cfg;
  const int H = cfg.n_heads, G = H / cfg.n_kv_heads;
  char* base = (char*)ws;
  aa->q = q; aa->seq_lens = seq_lens; aa->B = B; aa->T_cap = c.T_cap; aa->H = H;
  aa->n_kv = cfg.n_kv_heads; aa->dh = cfg.head_dim; aa->r = cfg.r_pairs; aa->d_c = cfg.d_c;
  aa->W_ukF = p.W_ukF;
  aa->rope_pair = p.rope_pair; aa->theta = p.theta;
  // f32 absorbed queries for the CUDA-core kernel, bf16 for the tensor-core kernels
  aa->qlat = L.kernel == 1 ? (float*)(base + L.off_qlat) : nullptr;
  aa->qlat16 = L.kernel != 1 ? (__nv_bfloat16*)(base + L.off_qlat) : nullptr;
  aa->qrope = (float*)(base + L.off_qrope);
  aa->sched = mla_sched_view(L, ws, B); aa->tile = L.tile; aa->G = L.G; aa->err = p.err;
  aa->sm_scale = cfg.softmax_scale > 0.0f ? cfg.softmax_scale : (float)(1.0 / sqrt((double)cfg.head_dim));
  aa->q_chunk = 1;
  aa->q_block = 1;
  {
    const int vecn = 16 / (int)sizeof(T);   // elements per 16-byte load
    aa->vec_ok = ((uintptr_t)q % 16 == 0) && cfg.d_c % vecn == 0 && cfg.head_dim % vecn == 0;
  }
  aa->mma = std::is_same<T, __nv_bfloat16>::value && aa->vec_ok && cfg.d_c % 8 == 0 && cfg.head_dim % 8 == 0;
  const int RPC = aa->mma ? kAbsRowsMma : kAbsRows;
  const int n_rb = (B * G + RPC - 1) / RPC, n_cc = (cfg.d_c + kAbsCols - 1) / kAbsCols;
  const int KP = (cfg.head_dim + 15) & ~15;
  const size_t smem_work =
      aa->mma ? sizeof(__nv_bfloat16) * ((size_t)KP * (kAbsCols + 8) + (size_t)kAbsRowsMma * (KP + 8))
              : sizeof(float) * ((size_t)cfg.head_dim * kAbsCols + (size_t)kAbsRows * cfg.head_dim);
  const size_t sched_ints = (size_t)9 * B + 4 * L.G + 2;
  *smem = std::min<size_t>(std::max(smem_work, sched_ints * sizeof(int32_t)), std::max<size_t>(smem_work, 160 * 1024));
  aa->sched_ints = (int)(*smem / sizeof(int32_t));
  *nblocks = cfg.n_kv_heads * n_rb * n_cc + 1;
}

// The split merge with W_uv over `units` merged units of H rows in n_kv row groups (decode:
// sequences, heads, KV heads; many queries per sequence: (sequence, query block) units of
// q_block * heads rows).
template <typename T>
cudaError_t launch_combine(const mla_plan& p, int units, int H, int n_kv, int q_chunk, int q_block, void* out,
                           void* ws, const DecodeLayout& L, const Sched& sched, cudaStream_t s) {
  const mla_config_t& cfg = p.cfg;
  char* base = (char*)ws;
  CombineArgs ca;
  ca.B = units; ca.H = H; ca.n_kv = n_kv; ca.d_c = cfg.d_c; ca.dh = cfg.head_dim;
  ca.opart = (const float*)(base + L.off_opart); ca.mlpart = (const float*)(base + L.off_mlpart);
  ca.sched = sched; ca.W_uv = p.W_uv; ca.out = out; ca.P = L.P;
  // many rows per W_uv group (a chunk of queries): more rows per CTA, fewer W stagings
  const int G = H / n_kv;
  ca.rpw = units * G >= 64 * kCmbRows ? kCmbMaxRpw : 1;
  const int RB = kCmbRows * ca.rpw, RBP = (RB + 15) & ~15;
  ca.ncols = (size_t)cfg.d_c * (64 + RB) * sizeof(float) <= 160 * 1024 ? 64 : 32;
  ca.vec_ok = cfg.head_dim % (16 / (int)sizeof(T)) == 0;
  ca.q_chunk = q_chunk; ca.q_block = q_block; ca.heads = cfg.n_heads;
  const size_t smem_c = (size_t)cfg.d_c * (ca.ncols + RB) * sizeof(float) +
                        (size_t)RBP * (cfg.d_c + 8) * sizeof(__nv_bfloat16);   // + the MMA form's A tiles
  const int n_rbc = (units * G + RB - 1) / RB, n_dc = (cfg.head_dim + ca.ncols - 1) / ca.ncols;
  cudaError_t e = cudaFuncSetAttribute(combine_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_c);
  if (e != cudaSuccess) return e;
  if ((e = mla_profile_event(p, kProfCombine, false, s)) != cudaSuccess) return e;
  e = mla_launch_kernel(combine_kernel<T>, dim3(n_kv * n_rbc * n_dc), dim3(256), smem_c, s, p.opt_pdl, ca);
  if (e != cudaSuccess) return e;
  return mla_profile_event(p, kProfCombine, true, s);
}

// Split-K attention over the latent cache, then the split merge with W_uv.
template <typename T, bool INT4>
cudaError_t launch_attention_combine(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, int B,
                                     void* out, void* ws, const DecodeLayout& L, const AbsorbArgs& aa, cudaStream_t s) {
  const mla_config_t& cfg = p.cfg;
  const int H = cfg.n_heads;
  char* base = (char*)ws;
  const Sched sched = aa.sched;
  cudaError_t e;
  if (L.kernel == 1) {
    DecodeArgs da;
    da.cache = c; da.seq_lens = seq_lens; da.err = p.err; da.qbits = mla_quant_bits(cfg.cache_kind); da.B = B; da.H = H; da.n_kv = cfg.n_kv_heads; da.r = cfg.r_pairs;
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
    if ((e = mla_profile_event(p, kProfAttention, false, s)) != cudaSuccess) return e;
    e = mla_launch_kernel(decode_simt_kernel<T, INT4>, dim3(L.G), dim3(256), smem, s, p.opt_pdl, da);
    if (e != cudaSuccess) return e;
    if ((e = mla_profile_event(p, kProfAttention, true, s)) != cudaSuccess) return e;
  } else if (L.kernel == 4) {
    e = mla_launch_chunk_tc(p, c, seq_lens, B, 1, sched, base + L.off_qlat, (const float*)(base + L.off_qrope),
                            (float*)(base + L.off_opart), (float*)(base + L.off_mlpart), L.P, L.G, s,
                            H <= 32 ? 32 : 128);
    if (e != cudaSuccess) return e;
  } else {
    e = mla_launch_decode_tc(p, c, seq_lens, B, sched, base + L.off_qlat, (const float*)(base + L.off_qrope),
                             (float*)(base + L.off_opart), (float*)(base + L.off_mlpart), L.P, L.G, s);
    if (e != cudaSuccess) return e;
  }
  return launch_combine<T>(p, B, H, cfg.n_kv_heads, 1, 1, out, ws, L, sched, s);
}

template <typename T, bool INT4>
cudaError_t launch_decode_t(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens,
                            const void* q, int B, void* out, void* ws, const DecodeLayout& L,
                            cudaStream_t s) {
  AbsorbArgs aa;
  size_t smem_abs;
  int nblk;
  absorb_setup<T>(p, c, seq_lens, q, B, ws, L, &aa, &smem_abs, &nblk);
  cudaError_t e = cudaFuncSetAttribute(absorb_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_abs);
  if (e != cudaSuccess) return e;
  if ((e = mla_profile_event(p, kProfAbsorb, false, s)) != cudaSuccess) return e;
  e = mla_launch_kernel(absorb_kernel<T>, dim3(nblk), dim3(256), smem_abs, s, p.opt_pdl, aa);
  if (e != cudaSuccess) return e;
  if ((e = mla_profile_event(p, kProfAbsorb, true, s)) != cudaSuccess) return e;
  return launch_attention_combine<T, INT4>(p, c, seq_lens, B, out, ws, L, aa, s);
}

// ------------------------------------------------------------ fused decode step
// The first kernel of a decode step: the append of every sequence's new token and the
// query absorption (with the split-K schedule) in one launch, as they depend on nothing
// of each other.  Blocks [0, n_abs) run the absorption grid (block 0, the schedule, is
// dispatched first), blocks [n_abs, n_abs + n_app) the append grid.
struct StepPreArgs {
  AbsorbArgs abs;
  AppendSmallArgs app;
  int n_abs, app_gx, app_gy;
};

template <bool INT4>
__global__ void __launch_bounds__(256, 1) step_pre_kernel(StepPreArgs sp) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int b = blockIdx.x;
  if (b < sp.n_abs) {
    absorb_body<__nv_bfloat16>(sp.abs, b, reinterpret_cast<float*>(smem));
  } else {
    const int k = b - sp.n_abs, gxy = sp.app_gx * sp.app_gy;
    append_small_mma_body<INT4>(sp.app, k % sp.app_gx, (k / sp.app_gx) % sp.app_gy, k / gxy, sp.app_gx, sp.app_gy,
                                smem);
  }
}

template <bool INT4>
cudaError_t launch_step_t(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, const void* x,
                          const void* q, int B, void* out, void* ws, const DecodeLayout& L, cudaStream_t s) {
  using bf16 = __nv_bfloat16;
  StepPreArgs sp;
  dim3 agrid;
  size_t smem_app = 0, smem_abs;
  int nabs;
  absorb_setup<bf16>(p, c, seq_lens, q, B, ws, L, &sp.abs, &smem_abs, &nabs);
  if (!mla_append_step_mma_form(p, x, seq_lens, B, c, &sp.app, &agrid, &smem_app)) {
    // no fused form for this shape: the append, then the decode, as separate launches
    cudaError_t e = mla_profile_event(p, kProfAppend, false, s);
    if (e == cudaSuccess) e = mla_launch_append_step(p, x, seq_lens, B, c, s);
    if (e == cudaSuccess) e = mla_profile_event(p, kProfAppend, true, s);
    if (e != cudaSuccess) return e;
    return launch_decode_t<bf16, INT4>(p, c, seq_lens, q, B, out, ws, L, s);
  }
  sp.n_abs = nabs;
  sp.app_gx = (int)agrid.x;
  sp.app_gy = (int)agrid.y;
  const int nblk = nabs + (int)(agrid.x * agrid.y * agrid.z);
  const size_t smem = std::max(smem_app, smem_abs);
  cudaError_t e = cudaFuncSetAttribute(step_pre_kernel<INT4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if ((e = mla_profile_event(p, kProfAbsorb, false, s)) != cudaSuccess) return e;
  e = mla_launch_kernel(step_pre_kernel<INT4>, dim3(nblk), dim3(256), smem, s, p.opt_pdl, sp);
  if (e != cudaSuccess) return e;
  if ((e = mla_profile_event(p, kProfAbsorb, true, s)) != cudaSuccess) return e;
  return launch_attention_combine<bf16, INT4>(p, c, seq_lens, B, out, ws, L, sp.abs, s);
}

// Many queries per sequence: absorption of every query (each rotated at its own position)
// with the schedule over (sequence, block of floor(128 / H) queries) units, the chunk
// attention kernel, and the merge of the units' rows.
cudaError_t launch_chunk(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, const void* q, int B,
                         int Q, void* out, void* ws, const DecodeLayout& L, cudaStream_t s) {
  using bf16 = __nv_bfloat16;
  const mla_config_t& cfg = p.cfg;
  const int kQB = 128 / cfg.n_heads;   // queries per unit: a unit holds up to 128 (query, head) rows
  AbsorbArgs aa;
  size_t smem_abs;
  int nblk;
  absorb_setup<bf16>(p, c, seq_lens, q, B * Q, ws, L, &aa, &smem_abs, &nblk);
  aa.q_chunk = Q;
  aa.q_block = kQB;
  cudaError_t e = cudaFuncSetAttribute(absorb_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_abs);
  if (e != cudaSuccess) return e;
  if ((e = mla_profile_event(p, kProfAbsorb, false, s)) != cudaSuccess) return e;
  e = mla_launch_kernel(absorb_kernel<bf16>, dim3(nblk), dim3(256), smem_abs, s, p.opt_pdl, aa);
  if (e != cudaSuccess) return e;
  if ((e = mla_profile_event(p, kProfAbsorb, true, s)) != cudaSuccess) return e;
  char* base = (char*)ws;
  const int units = B * ((Q + kQB - 1) / kQB);
  e = mla_launch_chunk_tc(p, c, seq_lens, B, Q, aa.sched, base + L.off_qlat, (const float*)(base + L.off_qrope),
                          (float*)(base + L.off_opart), (float*)(base + L.off_mlpart), L.P, L.G, s, 128);
  if (e != cudaSuccess) return e;
  return launch_combine<bf16>(p, units, kQB * cfg.n_heads, kQB * cfg.n_kv_heads, Q, kQB, out, ws, L, aa.sched, s);
}

}  // namespace mla

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

DecodeLayout mla_decode_layout(const mla_plan& p, int B, int kernel) {
  const mla_config_t& cfg = p.cfg;
  DecodeLayout L;
  L.kernel = kernel;
  L.tile = kernel == 2 ? 128 : kernel == 4 ? 64 : mla::kSimtTile;
  // the tensor-core kernels hold one CTA per SM (one wave); the CUDA-core kernel two
  L.G = p.opt_splits > 0 ? p.opt_splits : (kernel == 2 || kernel == 4 ? p.num_sms : 2 * p.num_sms);
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

DecodeLayout mla_chunk_layout(const mla_plan& p, int B, int Q) {
  const mla_config_t& cfg = p.cfg;
  DecodeLayout L;
  L.kernel = 3;
  L.tile = 64;
  L.G = p.opt_splits > 0 ? p.opt_splits : p.num_sms;
  const int qper = 128 / cfg.n_heads;   // queries per unit (see launch_chunk)
  const int units = B * ((Q + qper - 1) / qper), rows = qper * cfg.n_heads;
  L.P = units + L.G;
  L.K = cfg.d_c + p.R;
  const size_t nq = (size_t)B * Q * cfg.n_heads;   // query rows (query x head)
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align256(o + bytes); return r; };
  L.off_seq_tile0 = take(sizeof(int32_t) * units);
  L.off_seq_ntiles = take(sizeof(int32_t) * units);
  L.off_seq_ne = take(sizeof(int32_t) * (units + 1));
  L.off_seq_first = take(sizeof(int32_t) * units);
  L.off_seq_np = take(sizeof(int32_t) * units);
  L.off_worker_first = take(sizeof(int32_t) * (L.G + 1));
  L.off_piece_b = take(sizeof(int32_t) * L.P);
  L.off_piece_t0 = take(sizeof(int32_t) * L.P);
  L.off_piece_t1 = take(sizeof(int32_t) * L.P);
  L.off_qlat = take(sizeof(uint16_t) * nq * cfg.d_c);
  L.off_qrope = take(sizeof(float) * nq * 2 * cfg.r_pairs + 4);
  L.off_opart = take(sizeof(float) * (size_t)L.P * rows * cfg.d_c);
  L.off_mlpart = take(sizeof(float) * (size_t)L.P * rows * 2);
  L.total = o;
  return L;
}

cudaError_t mla_launch_chunk(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, const void* q,
                             int B, int Q, void* out, void* ws, const DecodeLayout& L, cudaStream_t s) {
  return mla::launch_chunk(p, c, seq_lens, q, B, Q, out, ws, L, s);
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
  const bool quant = mla_kind_quant(p.cfg.cache_kind);   // int4 or int2 codes
  if (p.cfg.dtype == MLA_BF16)
    return quant ? launch_decode_t<__nv_bfloat16, true>(p, c, seq_lens, q, B, out, ws, L, s)
                : launch_decode_t<__nv_bfloat16, false>(p, c, seq_lens, q, B, out, ws, L, s);
  return launch_decode_t<float, false>(p, c, seq_lens, q, B, out, ws, L, s);
}

cudaError_t mla_launch_step(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, const void* x,
                            const void* q, int B, void* out, void* ws, const DecodeLayout& L, cudaStream_t s) {
  using namespace mla;
  const bool quant = mla_kind_quant(p.cfg.cache_kind);
  if (p.cfg.dtype == MLA_BF16)
    return quant ? launch_step_t<true>(p, c, seq_lens, x, q, B, out, ws, L, s)
                 : launch_step_t<false>(p, c, seq_lens, x, q, B, out, ws, L, s);
  // float32: no fused form
  cudaError_t e = mla_profile_event(p, kProfAppend, false, s);
  if (e == cudaSuccess) e = mla_launch_append_step(p, x, seq_lens, B, c, s);
  if (e == cudaSuccess) e = mla_profile_event(p, kProfAppend, true, s);
  if (e != cudaSuccess) return e;
  return launch_decode_t<float, false>(p, c, seq_lens, q, B, out, ws, L, s);
}
