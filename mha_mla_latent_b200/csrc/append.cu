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
};

template <typename T, bool INT4>
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a) {
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

  // ---------------------------------------------------------------- epilogue
  const mla_cache_t& c = a.cache;
  // Column pairs: latent pairs (dtype cache) and RoPE pairs.
  for (int i = tid; i < kAppTokens * (kAppCols / 2); i += 256) {
    int t = i / (kAppCols / 2), cp = i % (kAppCols / 2);
    int n = tok0 + t, col = col0 + 2 * cp;
    if (n >= a.N || col >= a.ncols) continue;
    int sq = a.seq_idx[n], p = a.pos[n];
    if (sq < 0 || sq >= c.B || p < 0 || p >= c.T_cap) {
      if (col == 0) raise_error(a.err, MLA_DEVERR_APPEND_SLOT);
      continue;
    }
    size_t slot = (size_t)sq * c.T_cap + p;
    float v0 = red[t][2 * cp], v1 = red[t][2 * cp + 1];
    if (col < a.d_c) {
      if (!INT4) {
        T* dst = (T*)c.c_kv + slot * a.d_c + col;
        dst[0] = from_f32<T>(v0);
        dst[1] = from_f32<T>(v1);
      }
    } else {
      int rc = col - a.d_c;
      int g = rc / (2 * a.r), j = (rc % (2 * a.r)) / 2;
      int kpair = a.rope_pair[g * a.r + j];
      double sn, cs;
      sincos((double)p * a.theta[kpair], &sn, &cs);
      double o0 = (double)v0 * cs - (double)v1 * sn;
      double o1 = (double)v0 * sn + (double)v1 * cs;
      T* dst = (T*)c.k_rope + slot * a.R + rc;
      dst[0] = from_f64<T>(o0);
      dst[1] = from_f64<T>(o1);
    }
  }
  if (INT4) {
    // One warp per (token, 32-column group) of the latent.
    const int warp = tid / 32, lane = tid % 32;
    for (int w = warp; w < kAppTokens * (kAppCols / 32); w += 8) {
      int t = w / (kAppCols / 32), gi = w % (kAppCols / 32);
      int n = tok0 + t, col = col0 + gi * 32 + lane;
      if (n >= a.N || col0 + gi * 32 >= a.d_c) continue;   // whole group outside the latent
      int sq = a.seq_idx[n], p = a.pos[n];
      if (sq < 0 || sq >= c.B || p < 0 || p >= c.T_cap) continue;
      size_t slot = (size_t)sq * c.T_cap + p;
      float v = red[t][gi * 32 + lane];
      float am = fabsf(v);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      __half sh = __float2half_rn(__fdiv_rn(am, 7.0f));
      float sc = __half2float(sh);
      int code = 0;
      if (sc > 0.f) code = max(-7, min(7, (int)rintf(__fdiv_rn(v, sc))));
      uint32_t nib = (uint32_t)code & 15u;
      uint32_t hi = __shfl_down_sync(0xffffffffu, nib, 1);
      if ((lane & 1) == 0)
        ((uint8_t*)c.c_kv)[slot * (a.d_c / 2) + col / 2] = (uint8_t)(nib | (hi << 4));
      if (lane == 0) ((__half*)c.c_scales)[slot * (a.d_c / 32) + col / 32] = sh;
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

}  // namespace mla

cudaError_t mla_launch_append(const mla_plan& p, const void* x, const int32_t* seq_idx,
                              const int32_t* pos, int N, const mla_cache_t& c, cudaStream_t s) {
  using namespace mla;
  const mla_config_t& cfg = p.cfg;
  AppendArgs a;
  a.x = x; a.W = p.W_app; a.d = cfg.hidden; a.ncols = p.ncols; a.d_c = cfg.d_c; a.R = p.R;
  a.r = cfg.r_pairs; a.N = N; a.seq_idx = seq_idx; a.pos = pos; a.cache = c;
  a.rope_pair = p.rope_pair; a.theta = p.theta; a.err = p.err;
  // Split the hidden dim over a cluster when there are too few (token, column) tiles
  // to occupy the GPU; 8 is the portable cluster limit.
  int tiles = ((p.ncols + kAppCols - 1) / kAppCols) * ((N + kAppTokens - 1) / kAppTokens);
  int ksplit = 1;
  while (ksplit < 8 && tiles * ksplit * 2 <= p.num_sms && cfg.hidden / (ksplit * 2) >= 2 * kAppK)
    ksplit *= 2;
  int kslice = (cfg.hidden + ksplit - 1) / ksplit;
  kslice = (kslice + kAppK - 1) / kAppK * kAppK;
  a.kslice = kslice;
  bool int4 = cfg.cache_kind == MLA_CACHE_INT4_G32;
  if (cfg.dtype == MLA_BF16)
    return int4 ? launch_append_t<__nv_bfloat16, true>(a, ksplit, s)
                : launch_append_t<__nv_bfloat16, false>(a, ksplit, s);
  return launch_append_t<float, false>(a, ksplit, s);
}
