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

#include "append_common.cuh"

namespace cg = cooperative_groups;


namespace mla {

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
    int sq, p;
    append_slot(a, n, &sq, &p);
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
      float sn, cs;
      rope_sincos(p, a.theta[kpair], &sn, &cs);
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
      int sq, p;
      append_slot(a, n, &sq, &p);
      if (sq < 0 || sq >= c.B || p < 0 || p >= c.T_cap) continue;
      const MlaLoc lc = mla_loc(c, sq, p, a.err);
      const size_t slot = (size_t)lc.pb * lc.cap + lc.pt;
      const float v = tile[t * COLS + gi * 32 + lane];
      quant_group_store(c, slot, a.d_c, col, lane, v, a.qbits);
      const bool own = __shfl_sync(0xffffffffu, lane == 0 ? resid_owns(c, sq, p, a.step_lens != nullptr) : false, 0);
      if (own) resid_store(c, sq, p, a.d_c, col, v);
    }
  }
}

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
  // x and the token slots come from the caller, possibly from the kernel just before
  pdl_wait();
  pdl_trigger();

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
  // the token slots and x come from the caller, possibly from the kernel just before
  pdl_wait();
  pdl_trigger();
  if (tid < kSmTok) {
    append_slot(a, tok0 + tid, &s_sq[tid], &s_pos[tid]);
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

template <bool INT4>
__global__ void __launch_bounds__(256) append_small_mma_kernel(AppendSmallArgs sa) {
  extern __shared__ __align__(16) uint8_t sm8[];
  append_small_mma_body<INT4>(sa, blockIdx.x, blockIdx.y, blockIdx.z, gridDim.x, gridDim.y, sm8);
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

namespace {

mla::AppendArgs make_append_args(const mla_plan& p, const void* x, int N, const mla_cache_t& c) {
  const mla_config_t& cfg = p.cfg;
  mla::AppendArgs a;
  a.x = x; a.W = p.W_app; a.d = cfg.hidden; a.ncols = p.ncols; a.d_c = cfg.d_c; a.R = p.R;
  a.r = cfg.r_pairs; a.N = N; a.seq_idx = nullptr; a.pos = nullptr; a.cache = c;
  a.rope_pair = p.rope_pair; a.theta = p.theta; a.err = p.err; a.step_lens = nullptr;
  const size_t eb = cfg.dtype == MLA_BF16 ? 2 : 4;
  a.vec_ok = ((uintptr_t)x % 16 == 0) && ((size_t)cfg.hidden * eb) % 16 == 0 && ((size_t)p.ncols * eb) % 16 == 0;
  a.qbits = mla_quant_bits(cfg.cache_kind);
  a.kslice = 0;
  return a;
}

// The bf16 decode-step form (tensor-core slice products, ticket reduction), when it applies.
bool mma_form(const mla_plan& p, mla::AppendArgs a, mla::AppendSmallArgs* sa, dim3* grid, size_t* smem) {
  using namespace mla;
  const mla_config_t& cfg = p.cfg;
  if (!(a.N <= kAppMaxSmallTokens && p.app_part && p.app_ticket && cfg.dtype == MLA_BF16 && a.vec_ok)) return false;
  const int ks = (cfg.hidden + kAppSplit - 1) / kAppSplit;
  a.kslice = (ks + 127) / 128 * 128;
  if ((size_t)a.kslice * (kSmTok + kSmCols + 16) * 2 > 200 * 1024) return false;
  sa->a = a;
  sa->part = p.app_part;
  sa->ticket = p.app_ticket;
  *grid = dim3((a.ncols + kSmCols - 1) / kSmCols, (a.N + kSmTok - 1) / kSmTok, kAppSplit);
  *smem = std::max<size_t>(sizeof(__nv_bfloat16) * ((size_t)kSmTok * (a.kslice + 8) + (size_t)a.kslice * (kSmCols + 8)),
                           sizeof(float) * 8 * kSmTok * kSmCols);
  return true;
}

cudaError_t launch_append_args(const mla_plan& p, mla::AppendArgs a, const mla_cache_t& c, cudaStream_t s) {
  using namespace mla;
  const mla_config_t& cfg = p.cfg;
  const int N = a.N;
  const bool int4 = mla_kind_quant(cfg.cache_kind);   // quantised latent (int4 or int2 codes)
  if (c.c_resid && !a.step_lens) {   // residual window: claim the ring slots first
    const int grid = std::max(1, std::min((N + 255) / 256, 4 * p.num_sms));
    cudaError_t e =
        mla_launch_kernel(resid_claim_kernel, dim3(grid), dim3(256), 0, s, p.opt_pdl, a.seq_idx, a.pos, N, c);
    if (e != cudaSuccess) return e;
  }
  {
    AppendSmallArgs sa;
    dim3 grid;
    size_t smem;
    if (mma_form(p, a, &sa, &grid, &smem)) {
      auto kern = int4 ? append_small_mma_kernel<true> : append_small_mma_kernel<false>;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      return mla_launch_kernel(kern, grid, dim3(256), smem, s, p.opt_pdl, sa);
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

}  // namespace

bool mla_append_step_mma_form(const mla_plan& p, const void* x, const int32_t* seq_lens, int B,
                              const mla_cache_t& c, mla::AppendSmallArgs* sa, dim3* grid, size_t* smem) {
  mla::AppendArgs a = make_append_args(p, x, B, c);
  a.step_lens = seq_lens;
  return mma_form(p, a, sa, grid, smem);
}

cudaError_t mla_launch_append(const mla_plan& p, const void* x, const int32_t* seq_idx,
                              const int32_t* pos, int N, const mla_cache_t& c, cudaStream_t s) {
  mla::AppendArgs a = make_append_args(p, x, N, c);
  a.seq_idx = seq_idx;
  a.pos = pos;
  return launch_append_args(p, a, c, s);
}

cudaError_t mla_launch_append_step(const mla_plan& p, const void* x, const int32_t* seq_lens, int B,
                                   const mla_cache_t& c, cudaStream_t s) {
  mla::AppendArgs a = make_append_args(p, x, B, c);
  a.step_lens = seq_lens;
  return launch_append_args(p, a, c, s);
}
