// Cache append: c = x W_dkv and the RoPE key dims x W_krope, rotated at the token's
// position, optionally int4-quantised, scattered into the caller's cache.
//
// Paper notes "MHA2MLA" (ACL 2025), §关键设计: SVDjoint gives the down-projection
// W_dkv whose output c_kv is cached; partial-RoPE keeps each head's selected pairs,
// rotated at the token's position; §与 KV Cache 量化兼容: 4-bit quantisation of c_kv.
//
// One fused kernel.  A CTA computes a tile of 32 tokens x 64 packed columns
// ([W_dkv | W_krope]) over a slice of the hidden dim; when the token count is small the
// hidden dim is split across a thread-block cluster and the partial tiles are summed
// over distributed shared memory by the cluster's rank-0 CTA in fixed rank order
// (deterministic), which then runs the epilogue.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "warp_mma.cuh"

namespace cg = cooperative_groups;

MLA_KSPAN_DEFINE(append)

namespace mla {

constexpr int kAppTokens = 32;
constexpr int kAppCols = 64;
constexpr int kAppK = 32;

struct AppendArgs {
  const void* x;
  const void* W;            // [d][ncols]
  int d, ncols, d_c, R, r, N;
  const int32_t* seq_idx;
  const int32_t* pos;
  mla_cache_t cache;
  const int32_t* rope_pair;  // [n_kv][r]
  const double* theta;
  int32_t* err;
  int qbits;                // quantised latent (INT4 instantiations): code width, 4 or 2
  int kslice;               // hidden dims per cluster rank
  int vec_ok;               // x rows and W rows allow 16-byte vector loads
};

// Residual window (MLA_CACHE_INT4_G32_R128): the unquantised latent of token (sq, p), in
// the config dtype (bf16), goes to ring slot p % 128 when the slot is claimed by p (the
// claim kernel ran first and left there the largest position of the call for the slot).
__device__ __forceinline__ void resid_store(const mla_cache_t& c, int sq, int p, int d_c, int col, float v) {
  if (!c.c_resid) return;
  const size_t rs = (size_t)sq * MLA_RESID_WINDOW + (p & (MLA_RESID_WINDOW - 1));
  if (c.resid_pos[rs] == p) ((__nv_bfloat16*)c.c_resid)[rs * d_c + col] = __float2bfloat16_rn(v);
}

// Quantises one group of 32 latent values held one per lane (lane l: element col, the
// group's start + l) and stores codes and scale at token row `slot`.  4 bits: scale
// fp16(absmax/7), codes in [-7, 7], two per byte; 2 bits: scale fp16(absmax), codes in
// [-1, 1], four per byte.  Decisions in float32 (the division correctly rounded).
__device__ __forceinline__ void quant_group_store(const mla_cache_t& c, size_t slot, int d_c, int col, int lane,
                                                  float v, int qbits) {
  float am = fabsf(v);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const int qmax = qbits == 4 ? 7 : 1;
  const __half sh = __float2half_rn(qbits == 4 ? __fdiv_rn(am, 7.0f) : am);
  const float sc = __half2float(sh);
  int code = 0;
  if (sc > 0.f) code = max(-qmax, min(qmax, (int)rintf(__fdiv_rn(v, sc))));
  if (qbits == 4) {
    const uint32_t nib = (uint32_t)code & 15u;
    const uint32_t hi = __shfl_down_sync(0xffffffffu, nib, 1);
    if ((lane & 1) == 0) ((uint8_t*)c.c_kv)[slot * (d_c / 2) + col / 2] = (uint8_t)(nib | (hi << 4));
  } else {
    const uint32_t f = (uint32_t)code & 3u;
    const uint32_t f1 = __shfl_down_sync(0xffffffffu, f, 1), f2 = __shfl_down_sync(0xffffffffu, f, 2),
                   f3 = __shfl_down_sync(0xffffffffu, f, 3);
    if ((lane & 3) == 0) ((uint8_t*)c.c_kv)[slot * (d_c / 4) + col / 4] = (uint8_t)(f | (f1 << 2) | (f2 << 4) | (f3 << 6));
  }
  if (lane == 0) ((__half*)c.c_scales)[slot * (d_c / 32) + col / 32] = sh;
}

// Claims the residual ring slots of a call's tokens: resid_pos[seq][p % 128] becomes the
// largest position that maps there (an atomic maximum, so the newest token owns the slot
// whatever the order of the call's tokens).
__global__ void __launch_bounds__(256) resid_claim_kernel(const int32_t* __restrict__ seq_idx,
                                                          const int32_t* __restrict__ pos, int N,
                                                          mla_cache_t c) {
  pdl_wait();   // the kernel before may still read the ring
  pdl_trigger();
  for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < N; n += gridDim.x * blockDim.x) {
    const int sq = seq_idx[n], p = pos[n];
    if (sq < 0 || sq >= c.B || p < 0 || p >= c.T_cap) continue;   // reported by the append
    atomicMax(c.resid_pos + (size_t)sq * MLA_RESID_WINDOW + (p & (MLA_RESID_WINDOW - 1)), p);
  }
}

// Epilogue on a finished [TOK][COLS] tile of x [W_dkv | W_krope] sums held in shared
// memory: latent columns are stored in the cache encoding, RoPE columns are rotated at
// the token's position (angle in double) and stored; everything goes to (seq, pos).
template <typename T, bool INT4, int TOK, int COLS>
__device__ void append_epilogue(const AppendArgs& a, const float* tile, int tok0, int col0) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const mla_cache_t& c = a.cache;
  for (int i = tid; i < TOK * (COLS / 2); i += nt) {
    const int t = i / (COLS / 2), cp = i % (COLS / 2);
    const int n = tok0 + t, col = col0 + 2 * cp;
    if (n >= a.N || col >= a.ncols) continue;
    const int sq = a.seq_idx[n], p = a.pos[n];
    if (sq < 0 || sq >= c.B || p < 0 || p >= c.T_cap) {
      if (col == 0) raise_error(a.err, MLA_DEVERR_APPEND_SLOT);
      continue;
    }
    const MlaLoc lc = mla_loc(c, sq, p, a.err);
    const size_t slot = (size_t)lc.pb * lc.cap + lc.pt;
    const float v0 = tile[t * COLS + 2 * cp], v1 = tile[t * COLS + 2 * cp + 1];
    if (col < a.d_c) {
      if (!INT4) {
        T* dst = (T*)c.c_kv + slot * a.d_c + col;
        dst[0] = from_f32<T>(v0);
        dst[1] = from_f32<T>(v1);
      }
    } else {
      const int rc = col - a.d_c;
      const int g = rc / (2 * a.r), j = (rc % (2 * a.r)) / 2;
      const int kpair = a.rope_pair[g * a.r + j];
      double sn, cs;
      sincos((double)p * a.theta[kpair], &sn, &cs);
      T* dst = (T*)c.k_rope + mla_kr_offset(lc.pb, lc.pt, g, rc % (2 * a.r), lc.cap, a.R / (2 * a.r), 2 * a.r);
      dst[0] = from_f64<T>((double)v0 * cs - (double)v1 * sn);
      dst[1] = from_f64<T>((double)v0 * sn + (double)v1 * cs);
    }
  }
  if (INT4) {
    // One warp per (token, 32-column group) of the latent.
    const int warp = tid / 32, lane = tid % 32, nw = nt / 32;
    for (int w = warp; w < TOK * (COLS / 32); w += nw) {
      const int t = w / (COLS / 32), gi = w % (COLS / 32);
      const int n = tok0 + t, col = col0 + gi * 32 + lane;
      if (n >= a.N || col0 + gi * 32 >= a.d_c) continue;   // whole group outside the latent
      const int sq = a.seq_idx[n], p = a.pos[n];
      if (sq < 0 || sq >= c.B || p < 0 || p >= c.T_cap) continue;
      const MlaLoc lc = mla_loc(c, sq, p, a.err);
      const size_t slot = (size_t)lc.pb * lc.cap + lc.pt;
      const float v = tile[t * COLS + gi * 32 + lane];
      quant_group_store(c, slot, a.d_c, col, lane, v, a.qbits);
      resid_store(c, sq, p, a.d_c, col, v);
    }
  }
}

template <typename T, bool INT4>
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a) {
  MLA_KSPAN(1);
  __shared__ float xs[kAppTokens][kAppK + 1];
  __shared__ __align__(16) float ws[kAppK][kAppCols];
  __shared__ __align__(16) float red[kAppTokens][kAppCols];

  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;          // 4 columns x 2 tokens per thread
  const int col0 = blockIdx.x * kAppCols;
  const int tok0 = blockIdx.y * kAppTokens;
  const int rank = blockIdx.z;                     // == cluster rank (cluster spans z)
  const int nrank = gridDim.z;
  const int k_begin = rank * a.kslice;
  const int k_end = min(a.d, k_begin + a.kslice);
  const T* x = (const T*)a.x;
  const T* W = (const T*)a.W;

  float acc[2][4] = {};
  for (int k0 = k_begin; k0 < k_end; k0 += kAppK) {
    for (int i = tid; i < kAppTokens * kAppK; i += 256) {
      int t = i / kAppK, kk = i % kAppK;
      int n = tok0 + t, kd = k0 + kk;
      xs[t][kk] = (n < a.N && kd < k_end) ? to_f32(x[(size_t)n * a.d + kd]) : 0.f;
    }
    for (int i = tid; i < kAppK * kAppCols; i += 256) {
      int kk = i / kAppCols, c = i % kAppCols;
      int kd = k0 + kk, col = col0 + c;
      ws[kk][c] = (kd < k_end && col < a.ncols) ? to_f32(W[(size_t)kd * a.ncols + col]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kAppK; ++kk) {
      float x0 = xs[ty * 2][kk], x1 = xs[ty * 2 + 1][kk];
      float4 w = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
      acc[0][0] += x0 * w.x; acc[0][1] += x0 * w.y; acc[0][2] += x0 * w.z; acc[0][3] += x0 * w.w;
      acc[1][0] += x1 * w.x; acc[1][1] += x1 * w.y; acc[1][2] += x1 * w.z; acc[1][3] += x1 * w.w;
    }
    __syncthreads();
  }

  pdl_wait();   // the cache may still be read by the kernel before this one
  pdl_trigger();
  // Partial tile to shared memory; cluster reduction when the hidden dim is split.
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) red[ty * 2 + i][tx * 4 + j] = acc[i][j];
  if (nrank > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0) {
      for (int rr = 1; rr < nrank; ++rr) {
        float* remote = cluster.map_shared_rank(&red[0][0], rr);
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] += remote[(ty * 2 + i) * kAppCols + tx * 4 + j];
      }
    }
    cluster.sync();  // remote tiles stay alive until rank 0 has read them
    if (rank != 0) return;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) red[ty * 2 + i][tx * 4 + j] = acc[i][j];
  }
  __syncthreads();

  append_epilogue<T, INT4, kAppTokens, kAppCols>(a, &red[0][0], tok0, col0);
}

// Decode-step append (few tokens).  The product out[N][ncols] = x W_app is split into
// 32-token x 32-column tiles and kAppSplit slices of the hidden dim, one CTA each.  A CTA
// stages its x and W slices in one batch of loads, its eight warps each take an eighth of
// the slice with 8 x 4 register tiles, and the warps' tiles are summed in shared memory.
// The slice's partial tile goes to the plan's scratch; the last CTA of a tile to finish
// (ticket counter) sums the kAppSplit partials in slice order (deterministic) and runs the
// epilogue, whose per-token and per-column inputs every CTA prefetched at its start.
constexpr int kSmTok = 32, kSmCols = 32, kAppSplit = 8;

struct AppendSmallArgs {
  AppendArgs a;
  float* part;        // [kAppSplit][tiles][32 * 32] partial tiles
  int32_t* ticket;    // [tiles] arrival counters (the last CTA resets its counter)
};

// Second half of the decode-step append, after the eight warps' 32 x 32 tiles of this hidden-dim
// slice are in red[8][32 * 32]: sum them into the slice's partial, and let the last CTA of the
// tile sum the partials in slice order and write the cache (latent, RoPE keys rotated at the
// token's position, int4 codes).
template <typename T, bool INT4>
__device__ __forceinline__ void append_small_finish(const AppendSmallArgs& sa, float* red, const int* s_sq,
                                                    const int* s_pos, const double* s_theta, int* s_last,
                                                    int tok0, int col0, int tile, int ntile, int split) {
  const AppendArgs& a = sa.a;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the scratch and the cache may still be in use by the kernels before this one
  pdl_wait();
  pdl_trigger();
  float* my_part = sa.part + ((size_t)split * ntile + tile) * (kSmTok * kSmCols);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int o = tid + 256 * e;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[w * kSmTok * kSmCols + o];
    my_part[o] = v;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(sa.ticket + tile, 1);
    *s_last = prev == kAppSplit - 1;
    if (*s_last) sa.ticket[tile] = 0;   // ready for the next call
  }
  __syncthreads();
  if (!*s_last) return;
  __threadfence();
  // ---- last CTA of the tile: sum the partials in slice order, then the epilogue
  float* tileb = red;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int o = tid + 256 * e;
    float v = 0.f;
    for (int sp = 0; sp < kAppSplit; ++sp) v += __ldcg(sa.part + ((size_t)sp * ntile + tile) * (kSmTok * kSmCols) + o);
    tileb[o] = v;
  }
  __syncthreads();
  const mla_cache_t& c = a.cache;
  const int n_kv = a.R / max(2 * a.r, 1);
  for (int i = tid; i < kSmTok * (kSmCols / 2); i += 256) {
    const int t = i / (kSmCols / 2), cp = i % (kSmCols / 2);
    const int n = tok0 + t, col = col0 + 2 * cp;
    if (n >= a.N || col >= a.ncols) continue;
    const int sq = s_sq[t], p = s_pos[t];
    if (sq < 0 || sq >= c.B || p < 0 || p >= c.T_cap) {
      if (col == 0) raise_error(a.err, MLA_DEVERR_APPEND_SLOT);
      continue;
    }
    const float v0 = tileb[t * kSmCols + 2 * cp], v1 = tileb[t * kSmCols + 2 * cp + 1];
    const MlaLoc lc = mla_loc(c, sq, p, a.err);
    if (col < a.d_c) {
      if (!INT4) {
        T* dst = (T*)c.c_kv + ((size_t)lc.pb * lc.cap + lc.pt) * a.d_c + col;
        dst[0] = from_f32<T>(v0);
        dst[1] = from_f32<T>(v1);
      }
    } else {
      const int rc = col - a.d_c;
      double sn, cs;
      sincos((double)p * s_theta[cp], &sn, &cs);
      T* dst = (T*)c.k_rope + mla_kr_offset(lc.pb, lc.pt, rc / (2 * a.r), rc % (2 * a.r), lc.cap, n_kv, 2 * a.r);
      dst[0] = from_f64<T>((double)v0 * cs - (double)v1 * sn);
      dst[1] = from_f64<T>((double)v0 * sn + (double)v1 * cs);
    }
  }
  if (INT4 && col0 < a.d_c) {
    // one warp per token: the tile's 32 latent columns are one quantisation group
    for (int t = warp; t < kSmTok; t += 8) {
      const int n = tok0 + t;
      const int sq = s_sq[t], p = s_pos[t];
      if (n >= a.N || sq < 0 || sq >= c.B || p < 0 || p >= c.T_cap) continue;
      const MlaLoc lc = mla_loc(c, sq, p, a.err);
      const size_t slot = (size_t)lc.pb * lc.cap + lc.pt;
      const float v = tileb[t * kSmCols + lane];
      quant_group_store(c, slot, a.d_c, col0 + lane, lane, v, a.qbits);
      resid_store(c, sq, p, a.d_c, col0 + lane, v);
    }
  }
}

template <typename T, bool INT4>
cudaError_t launch_append_t(const AppendArgs& args, int ksplit, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((args.ncols + kAppCols - 1) / kAppCols, (args.N + kAppTokens - 1) / kAppTokens,
                     ksplit);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = ksplit;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, append_kernel<T, INT4>, args);
}

template <typename T, bool INT4>
__global__ void __launch_bounds__(256) append_small_kernel(AppendSmallArgs sa) {
  MLA_KSPAN(0);
  const AppendArgs& a = sa.a;
  extern __shared__ __align__(16) float smf[];
  const int ks = a.kslice;                       // multiple of 64
  float* xs = smf;                               // [ks][kSmTok]   (k-major)
  float* ws = xs + ks * kSmTok;                  // [ks][kSmCols]
  float* red = xs;                               // [8][kSmTok * kSmCols], after the product
  __shared__ int s_sq[kSmTok], s_pos[kSmTok];
  __shared__ double s_theta[kSmCols / 2];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int col0 = blockIdx.x * kSmCols, tok0 = blockIdx.y * kSmTok;
  const int split = blockIdx.z;
  const int tile = blockIdx.y * gridDim.x + blockIdx.x, ntile = gridDim.x * gridDim.y;
  const int k_begin = split * ks, k_end = min(a.d, k_begin + ks);
  const T* x = (const T*)a.x;
  const T* W = (const T*)a.W;
  constexpr int VEC = 16 / sizeof(T);
  // ---- epilogue inputs (token slots, rotation frequencies), prefetched
  if (tid < kSmTok) {
    const int n = tok0 + tid;
    s_sq[tid] = n < a.N ? __ldg(a.seq_idx + n) : -1;
    s_pos[tid] = n < a.N ? __ldg(a.pos + n) : -1;
  } else if (tid < kSmTok + kSmCols / 2) {
    const int cp = tid - kSmTok, col = col0 + 2 * cp;
    double th = 0.0;
    if (col >= a.d_c && col < a.ncols) {
      const int rc = col - a.d_c, g = rc / (2 * a.r), j = (rc % (2 * a.r)) / 2;
      th = __ldg(a.theta + __ldg(a.rope_pair + g * a.r + j));
    }
    s_theta[cp] = th;
  }
  // ---- x slice -> xs[k][t] and W slice -> ws[k][c]: 8 loads per thread in flight
  {
    const int nxv = kSmTok * (ks / VEC), nwv = ks * (kSmCols / VEC);
    for (int base = 0; base < nxv + nwv; base += 8 * 256) {
      uint4 r[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int v = base + tid + 256 * k;
        r[k] = make_uint4(0, 0, 0, 0);
        if (v < nxv) {
          const int t = v % kSmTok, ch = v / kSmTok;
          const int n = tok0 + t, kd = k_begin + ch * VEC;
          if (n < a.N && kd + VEC <= k_end && a.vec_ok)
            r[k] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)n * a.d + kd));
        } else if (v < nxv + nwv) {
          const int vw = v - nxv;
          const int kk = vw / (kSmCols / VEC), part = vw % (kSmCols / VEC);
          const int kd = k_begin + kk, col = col0 + part * VEC;
          if (kd < k_end && col + VEC <= a.ncols && a.vec_ok)
            r[k] = __ldg(reinterpret_cast<const uint4*>(W + (size_t)kd * a.ncols + col));
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int v = base + tid + 256 * k;
        float f[VEC];
        const T* e = reinterpret_cast<const T*>(&r[k]);
        if (v < nxv) {
          const int t = v % kSmTok, ch = v / kSmTok;
          const int n = tok0 + t, kd = k_begin + ch * VEC;
          const bool whole = n < a.N && kd + VEC <= k_end && a.vec_ok;
#pragma unroll
          for (int q = 0; q < VEC; ++q)
            f[q] = whole ? to_f32(e[q]) : ((n < a.N && kd + q < k_end) ? ldg_f32(x + (size_t)n * a.d + kd + q) : 0.f);
#pragma unroll
          for (int q = 0; q < VEC; ++q) xs[(ch * VEC + q) * kSmTok + t] = f[q];
        } else if (v < nxv + nwv) {
          const int vw = v - nxv;
          const int kk = vw / (kSmCols / VEC), part = vw % (kSmCols / VEC);
          const int kd = k_begin + kk, col = col0 + part * VEC;
          const bool whole = kd < k_end && col + VEC <= a.ncols && a.vec_ok;
#pragma unroll
          for (int q = 0; q < VEC; ++q)
            f[q] = whole ? to_f32(e[q])
                         : ((kd < k_end && col + q < a.ncols) ? ldg_f32(W + (size_t)kd * a.ncols + col + q) : 0.f);
#pragma unroll
          for (int q = 0; q < VEC; ++q) ws[kk * kSmCols + part * VEC + q] = f[q];
        }
      }
    }
  }
  __syncthreads();
  // ---- product: warp w takes hidden dims [w ks/8, (w+1) ks/8); lane -> 8 tokens x 4 columns
  const int tg = lane >> 3, cg = lane & 7;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  const int kw = ks / 8;
#pragma unroll 4
  for (int kk = warp * kw; kk < (warp + 1) * kw; ++kk) {
    const float4 x0 = *reinterpret_cast<const float4*>(&xs[kk * kSmTok + 8 * tg]);
    const float4 x1 = *reinterpret_cast<const float4*>(&xs[kk * kSmTok + 8 * tg + 4]);
    const float4 wv = *reinterpret_cast<const float4*>(&ws[kk * kSmCols + 4 * cg]);
    const float xa[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w}, wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += xa[i] * wa[j];
  }
  __syncthreads();   // xs is reused for the warps' tiles
#pragma unroll
  for (int i = 0; i < 8; ++i)
    *reinterpret_cast<float4*>(&red[warp * kSmTok * kSmCols + (8 * tg + i) * kSmCols + 4 * cg]) =
        make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
  __syncthreads();
  append_small_finish<T, INT4>(sa, red, s_sq, s_pos, s_theta, &s_last, tok0, col0, tile, ntile, split);
}

// bf16 form of the decode-step append: the slice product runs on the tensor cores as
// m16n8k16 warp MMAs from bf16 tiles staged with cp.async (x [32][ks], W [ks][32], rows
// padded by 16 bytes so the ldmatrix reads are conflict-free); warp w takes hidden dims
// [w ks/8, (w+1) ks/8) for the whole 32 x 32 tile.
template <bool INT4>
__global__ void __launch_bounds__(256) append_small_mma_kernel(AppendSmallArgs sa) {
  MLA_KSPAN(2);
  using bf16 = __nv_bfloat16;
  const AppendArgs& a = sa.a;
  extern __shared__ __align__(16) uint8_t sm8[];
  const int ks = a.kslice;                       // multiple of 128
  const int XLD = ks + 8;
  constexpr int WLD = kSmCols + 8;
  bf16* xs = reinterpret_cast<bf16*>(sm8);       // [kSmTok][XLD]
  bf16* wsm = xs + kSmTok * XLD;                 // [ks][WLD]
  float* red = reinterpret_cast<float*>(sm8);    // [8][kSmTok * kSmCols], after the product
  __shared__ int s_sq[kSmTok], s_pos[kSmTok];
  __shared__ double s_theta[kSmCols / 2];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int col0 = blockIdx.x * kSmCols, tok0 = blockIdx.y * kSmTok;
  const int split = blockIdx.z;
  const int tile = blockIdx.y * gridDim.x + blockIdx.x, ntile = gridDim.x * gridDim.y;
  const int k_begin = split * ks, k_end = min(a.d, k_begin + ks);
  const bf16* x = (const bf16*)a.x;
  const bf16* W = (const bf16*)a.W;
  if (tid < kSmTok) {
    const int n = tok0 + tid;
    s_sq[tid] = n < a.N ? __ldg(a.seq_idx + n) : -1;
    s_pos[tid] = n < a.N ? __ldg(a.pos + n) : -1;
  } else if (tid < kSmTok + kSmCols / 2) {
    const int cp = tid - kSmTok, col = col0 + 2 * cp;
    double th = 0.0;
    if (col >= a.d_c && col < a.ncols) {
      const int rc = col - a.d_c, g = rc / (2 * a.r), j = (rc % (2 * a.r)) / 2;
      th = __ldg(a.theta + __ldg(a.rope_pair + g * a.r + j));
    }
    s_theta[cp] = th;
  }
  // ---- stage: 16-byte asynchronous copies, all in flight together (missing rows and
  // columns are zero-filled)
  {
    const int nxv = kSmTok * (ks / 8), nwv = ks * (kSmCols / 8);
    for (int v = tid; v < nxv + nwv; v += 256) {
      if (v < nxv) {
        const int t = v / (ks / 8), ch = v % (ks / 8);
        const int n = tok0 + t, kd = k_begin + ch * 8;
        const bool ok = n < a.N && kd + 8 <= k_end;
        sm100::cp_async16(wmma16::smem_addr(xs + t * XLD + ch * 8), ok ? (const void*)(x + (size_t)n * a.d + kd) : a.x,
                          ok ? 16u : 0u);
      } else {
        const int vw = v - nxv;
        const int kk = vw / (kSmCols / 8), part = vw % (kSmCols / 8);
        const int kd = k_begin + kk, col = col0 + part * 8;
        const bool ok = kd < k_end && col + 8 <= a.ncols;
        sm100::cp_async16(wmma16::smem_addr(wsm + kk * WLD + part * 8),
                          ok ? (const void*)(W + (size_t)kd * a.ncols + col) : a.W, ok ? 16u : 0u);
      }
    }
    sm100::cp_async_commit();
    sm100::cp_async_wait_all();
  }
  __syncthreads();
  float acc[2][4][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
  const int kw = ks / 8;
  for (int k0 = warp * kw; k0 < (warp + 1) * kw; k0 += 16) {
    uint32_t a0[4], a1[4], b0[4], b1[4];
    wmma16::load_a(a0, xs, XLD, 0, k0, lane);
    wmma16::load_a(a1, xs, XLD, 16, k0, lane);
    wmma16::load_b2(b0, wsm, WLD, k0, 0, lane);
    wmma16::load_b2(b1, wsm, WLD, k0, 16, lane);
    wmma16::mma_16816(acc[0][0], a0, b0[0], b0[1]);
    wmma16::mma_16816(acc[0][1], a0, b0[2], b0[3]);
    wmma16::mma_16816(acc[0][2], a0, b1[0], b1[1]);
    wmma16::mma_16816(acc[0][3], a0, b1[2], b1[3]);
    wmma16::mma_16816(acc[1][0], a1, b0[0], b0[1]);
    wmma16::mma_16816(acc[1][1], a1, b0[2], b0[3]);
    wmma16::mma_16816(acc[1][2], a1, b1[0], b1[1]);
    wmma16::mma_16816(acc[1][3], a1, b1[2], b1[3]);
  }
  __syncthreads();   // the staging area is reused for the warps' tiles
  float* my = red + warp * kSmTok * kSmCols;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = 16 * i + (lane >> 2), col = 8 * j + 2 * (lane & 3);
      *reinterpret_cast<float2*>(my + row * kSmCols + col) = make_float2(acc[i][j][0], acc[i][j][1]);
      *reinterpret_cast<float2*>(my + (row + 8) * kSmCols + col) = make_float2(acc[i][j][2], acc[i][j][3]);
    }
  __syncthreads();
  append_small_finish<bf16, INT4>(sa, red, s_sq, s_pos, s_theta, &s_last, tok0, col0, tile, ntile, split);
}

template <bool INT4>
cudaError_t launch_append_small_mma(const AppendSmallArgs& sa, cudaStream_t s, bool pdl) {
  const AppendArgs& a = sa.a;
  dim3 grid((a.ncols + kSmCols - 1) / kSmCols, (a.N + kSmTok - 1) / kSmTok, kAppSplit);
  const size_t smem = std::max<size_t>(sizeof(__nv_bfloat16) * ((size_t)kSmTok * (a.kslice + 8) +
                                                                (size_t)a.kslice * (kSmCols + 8)),
                                       sizeof(float) * 8 * kSmTok * kSmCols);
  cudaError_t e = cudaFuncSetAttribute(append_small_mma_kernel<INT4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  return mla_launch_kernel(append_small_mma_kernel<INT4>, grid, dim3(256), smem, s, pdl, sa);
}

template <typename T, bool INT4>
cudaError_t launch_append_small_t(const AppendSmallArgs& sa, size_t smem, cudaStream_t s, bool pdl) {
  const AppendArgs& a = sa.a;
  dim3 grid((a.ncols + kSmCols - 1) / kSmCols, (a.N + kSmTok - 1) / kSmTok, kAppSplit);
  cudaError_t e = cudaFuncSetAttribute(append_small_kernel<T, INT4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  return mla_launch_kernel(append_small_kernel<T, INT4>, grid, dim3(256), smem, s, pdl, sa);
}

}  // namespace mla

cudaError_t mla_launch_append(const mla_plan& p, const void* x, const int32_t* seq_idx,
                              const int32_t* pos, int N, const mla_cache_t& c, cudaStream_t s) {
  using namespace mla;
  const mla_config_t& cfg = p.cfg;
  AppendArgs a;
  a.x = x; a.W = p.W_app; a.d = cfg.hidden; a.ncols = p.ncols; a.d_c = cfg.d_c; a.R = p.R;
  a.r = cfg.r_pairs; a.N = N; a.seq_idx = seq_idx; a.pos = pos; a.cache = c;
  a.rope_pair = p.rope_pair; a.theta = p.theta; a.err = p.err;
  const size_t eb = cfg.dtype == MLA_BF16 ? 2 : 4;
  a.vec_ok = ((uintptr_t)x % 16 == 0) && ((size_t)cfg.hidden * eb) % 16 == 0 && ((size_t)p.ncols * eb) % 16 == 0;
  const bool int4 = mla_kind_quant(cfg.cache_kind);   // quantised latent (int4 or int2 codes)
  a.qbits = mla_quant_bits(cfg.cache_kind);
  if (c.c_resid) {   // residual window: claim the ring slots first
    const int grid = std::max(1, std::min((N + 255) / 256, 4 * p.num_sms));
    cudaError_t e = mla_launch_kernel(resid_claim_kernel, dim3(grid), dim3(256), 0, s, p.opt_pdl, seq_idx, pos, N, c);
    if (e != cudaSuccess) return e;
  }
  if (N <= kAppMaxSmallTokens && p.app_part && p.app_ticket && cfg.dtype == MLA_BF16 && a.vec_ok) {
    int ks = (cfg.hidden + kAppSplit - 1) / kAppSplit;
    a.kslice = (ks + 127) / 128 * 128;
    if ((size_t)a.kslice * (kSmTok + kSmCols + 16) * 2 <= 200 * 1024) {
      AppendSmallArgs sa;
      sa.a = a;
      sa.part = p.app_part;
      sa.ticket = p.app_ticket;
      return int4 ? launch_append_small_mma<true>(sa, s, p.opt_pdl) : launch_append_small_mma<false>(sa, s, p.opt_pdl);
    }
  }
  if (N <= kAppMaxSmallTokens && p.app_part && p.app_ticket) {
    // decode-step size: kAppSplit slices of the hidden dim, 32 x 32 tiles
    int ks = (cfg.hidden + kAppSplit - 1) / kAppSplit;
    a.kslice = (ks + 63) / 64 * 64;
    // x and W slices, later reused for the eight warps' 32 x 32 tiles
    const size_t smem = sizeof(float) * std::max<size_t>((size_t)a.kslice * (kSmTok + kSmCols), 8 * kSmTok * kSmCols);
    if (smem <= 200 * 1024) {
      AppendSmallArgs sa;
      sa.a = a;
      sa.part = p.app_part;
      sa.ticket = p.app_ticket;
      if (cfg.dtype == MLA_BF16)
        return int4 ? launch_append_small_t<__nv_bfloat16, true>(sa, smem, s, p.opt_pdl)
                    : launch_append_small_t<__nv_bfloat16, false>(sa, smem, s, p.opt_pdl);
      return launch_append_small_t<float, false>(sa, smem, s, p.opt_pdl);
    }
  }
  // Split the hidden dim over a cluster when there are too few (token, column) tiles
  // to occupy the GPU; 8 is the portable cluster limit.
  int tiles = ((p.ncols + kAppCols - 1) / kAppCols) * ((N + kAppTokens - 1) / kAppTokens);
  int ksplit = 1;
  while (ksplit < 8 && tiles * ksplit * 2 <= p.num_sms && cfg.hidden / (ksplit * 2) >= 2 * kAppK)
    ksplit *= 2;
  int kslice = (cfg.hidden + ksplit - 1) / ksplit;
  kslice = (kslice + kAppK - 1) / kAppK * kAppK;
  a.kslice = kslice;
  if (cfg.dtype == MLA_BF16)
    return int4 ? launch_append_t<__nv_bfloat16, true>(a, ksplit, s)
                : launch_append_t<__nv_bfloat16, false>(a, ksplit, s);
  return launch_append_t<float, false>(a, ksplit, s);
}
