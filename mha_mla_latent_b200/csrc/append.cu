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

#include "common.cuh"

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
  int kslice;               // hidden dims per cluster rank
  int vec_ok;               // x rows and W rows allow 16-byte vector loads
};

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
    const size_t slot = (size_t)sq * c.T_cap + p;
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
      T* dst = (T*)c.k_rope + mla_kr_offset(sq, p, g, rc % (2 * a.r), c.T_cap, a.R / (2 * a.r), 2 * a.r);
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
      const size_t slot = (size_t)sq * c.T_cap + p;
      const float v = tile[t * COLS + gi * 32 + lane];
      float am = fabsf(v);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      const __half sh = __float2half_rn(__fdiv_rn(am, 7.0f));
      const float sc = __half2float(sh);
      int code = 0;
      if (sc > 0.f) code = max(-7, min(7, (int)rintf(__fdiv_rn(v, sc))));
      const uint32_t nib = (uint32_t)code & 15u;
      const uint32_t hi = __shfl_down_sync(0xffffffffu, nib, 1);
      if ((lane & 1) == 0) ((uint8_t*)c.c_kv)[slot * (a.d_c / 2) + col / 2] = (uint8_t)(nib | (hi << 4));
      if (lane == 0) ((__half*)c.c_scales)[slot * (a.d_c / 32) + col / 32] = sh;
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

// Decode-step append (few tokens): a CTA computes 32 tokens x 32 packed columns over one
// eighth of the hidden dim.  It loads its whole x and W slices up front (16-byte vector
// loads, all in flight together), accumulates 4x4 register tiles in four hidden-dim
// groups, and the eight CTAs of the cluster sum their tiles over distributed shared
// memory (fixed rank order) before rank 0 runs the epilogue.
constexpr int kSmTok = 32, kSmCols = 32, kSmSplit = 8;

template <typename T, bool INT4>
__global__ void __launch_bounds__(256) append_small_kernel(AppendArgs a) {
  MLA_KSPAN(0);
  extern __shared__ __align__(16) float smf[];
  const int ks = a.kslice;                       // multiple of 32
  float* xs = smf;                               // [ks][kSmTok]   (k-major)
  float* ws = xs + ks * kSmTok;                  // [ks][kSmCols]
  float* red = ws + ks * kSmCols;                // [4][kSmTok][kSmCols]
  const int tid = threadIdx.x;
  const int col0 = blockIdx.x * kSmCols, tok0 = blockIdx.y * kSmTok;
  const int rank = blockIdx.z;
  const int k_begin = rank * ks, k_end = min(a.d, k_begin + ks);
  const T* x = (const T*)a.x;
  const T* W = (const T*)a.W;
  constexpr int VEC = 16 / sizeof(T);
  // x slice [32 tokens][ks] and W slice [ks][32 columns]: batches of eight 16-byte loads per
  // thread are all issued before any is stored, so each batch costs one memory round trip.
  // x: consecutive threads take consecutive tokens so the transposed stores do not collide.
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
  __syncthreads();
  // 4 hidden-dim groups x (8 token quads x 8 column quads)
  const int kg = tid / 64, tt = (tid % 64) / 8, cc = tid % 8;
  float acc[4][4] = {};
  const int kq = ks / 4;
#pragma unroll 4
  for (int kk = kg * kq; kk < (kg + 1) * kq; ++kk) {
    const float4 xv = *reinterpret_cast<const float4*>(&xs[kk * kSmTok + tt * 4]);
    const float4 wv = *reinterpret_cast<const float4*>(&ws[kk * kSmCols + cc * 4]);
    const float xa[4] = {xv.x, xv.y, xv.z, xv.w}, wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += xa[i] * wa[j];
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) red[(kg * kSmTok + tt * 4 + i) * kSmCols + cc * 4 + j] = acc[i][j];
  __syncthreads();
  float* tile = red;   // group sums into group 0's slot
  for (int i = tid; i < kSmTok * kSmCols; i += 256)
    tile[i] = red[i] + red[kSmTok * kSmCols + i] + red[2 * kSmTok * kSmCols + i] + red[3 * kSmTok * kSmCols + i];
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  float fin[kSmTok * kSmCols / 256];
  if (rank == 0) {
#pragma unroll
    for (int e = 0; e < kSmTok * kSmCols / 256; ++e) fin[e] = tile[tid + 256 * e];
    for (int rr = 1; rr < (int)gridDim.z; ++rr) {
      const float* remote = cluster.map_shared_rank(tile, rr);
#pragma unroll
      for (int e = 0; e < kSmTok * kSmCols / 256; ++e) fin[e] += remote[tid + 256 * e];
    }
  }
  cluster.sync();  // remote tiles stay alive until rank 0 has read them
  if (rank != 0) return;
#pragma unroll
  for (int e = 0; e < kSmTok * kSmCols / 256; ++e) tile[tid + 256 * e] = fin[e];
  __syncthreads();
  append_epilogue<T, INT4, kSmTok, kSmCols>(a, tile, tok0, col0);
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
cudaError_t launch_append_small_t(const AppendArgs& args, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((args.ncols + kSmCols - 1) / kSmCols, (args.N + kSmTok - 1) / kSmTok, kSmSplit);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = sizeof(float) * ((size_t)args.kslice * (kSmTok + kSmCols) + 4 * kSmTok * kSmCols);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = kSmSplit;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaFuncSetAttribute(append_small_kernel<T, INT4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)cfg.dynamicSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, append_small_kernel<T, INT4>, args);
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
  const bool int4 = cfg.cache_kind == MLA_CACHE_INT4_G32;
  if (N <= 4 * kSmTok) {
    // decode-step size: split the hidden dim over an 8-CTA cluster, 32-column tiles
    int ks = (cfg.hidden + kSmSplit - 1) / kSmSplit;
    a.kslice = (ks + 31) / 32 * 32;
    if (sizeof(float) * ((size_t)a.kslice * (kSmTok + kSmCols) + 4 * kSmTok * kSmCols) <= 200 * 1024) {
      if (cfg.dtype == MLA_BF16)
        return int4 ? launch_append_small_t<__nv_bfloat16, true>(a, s)
                    : launch_append_small_t<__nv_bfloat16, false>(a, s);
      return launch_append_small_t<float, false>(a, s);
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
