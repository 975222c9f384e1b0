// 2-norm pair scores and head-wise top-r selection (conversion time).
//
// Paper notes "MHA2MLA" (ACL 2025), §关键设计, contribution-aware partial-RoPE
// removal: the contribution of frequency subspace [2k,2k+1] to the attention score is
// bounded by ||q^[2k,2k+1]|| * ||k^[2k,2k+1]||; the score is that bound averaged over
// calibration tokens (and over the query heads sharing a KV head), and each head keeps
// the r pairs with the largest score.  One CTA per KV head; float32 accumulation in a
// fixed order, so the result is deterministic.
#include "common.cuh"

namespace mla {

template <typename T>
__global__ void __launch_bounds__(256)
select_pairs_kernel(const T* __restrict__ q, const T* __restrict__ k, int T_, int H, int n_kv,
                    int dh, int r, int32_t* __restrict__ pair_idx, float* __restrict__ contrib) {
  const int g = blockIdx.x;
  const int P = dh / 2;
  const int G = H / n_kv;
  const int lanes = blockDim.x / P;          // token lanes per pair
  const int kk = threadIdx.x % P;
  const int lane = threadIdx.x / P;
  __shared__ float part[256];
  __shared__ float score[128];
  float acc = 0.f;
  if (lane < lanes) {
    for (int t = lane; t < T_; t += lanes) {
      const T* kp = k + ((size_t)t * n_kv + g) * dh + 2 * kk;
      float ka = to_f32(kp[0]), kb = to_f32(kp[1]);
      float kn = sqrtf(ka * ka + kb * kb);
      float qs = 0.f;
      for (int h = g * G; h < (g + 1) * G; ++h) {
        const T* qp = q + ((size_t)t * H + h) * dh + 2 * kk;
        float qa = to_f32(qp[0]), qb = to_f32(qp[1]);
        qs += sqrtf(qa * qa + qb * qb);
      }
      acc += qs * kn;
    }
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < P) {
    float s = 0.f;
    for (int l = 0; l < lanes; ++l) s += part[l * P + threadIdx.x];
    s = s / ((float)T_ * (float)G);
    score[threadIdx.x] = s;
    if (contrib) contrib[g * P + threadIdx.x] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // top-r: repeatedly take the largest unselected score, lower index on ties
    uint64_t taken0 = 0, taken1 = 0;  // P <= 128
    for (int j = 0; j < r; ++j) {
      int best = -1;
      float bv = 0.f;
      for (int i = 0; i < P; ++i) {
        bool t = (i < 64) ? ((taken0 >> i) & 1ull) : ((taken1 >> (i - 64)) & 1ull);
        if (t) continue;
        if (best < 0 || score[i] > bv) { best = i; bv = score[i]; }
      }
      if (best < 64) taken0 |= 1ull << best; else taken1 |= 1ull << (best - 64);
    }
    int n = 0;
    for (int i = 0; i < P; ++i) {
      bool t = (i < 64) ? ((taken0 >> i) & 1ull) : ((taken1 >> (i - 64)) & 1ull);
      if (t) pair_idx[g * r + (n++)] = i;
    }
  }
}

}  // namespace mla

cudaError_t mla_launch_select_pairs(const mla_config_t& cfg, const void* q, const void* k, int T,
                                    int32_t* pair_idx, float* contrib, cudaStream_t s) {
  dim3 grid(cfg.n_kv_heads), block(256);
  if (cfg.dtype == MLA_BF16)
    mla::select_pairs_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, T, cfg.n_heads, cfg.n_kv_heads,
        cfg.head_dim, cfg.r_pairs, pair_idx, contrib);
  else
    mla::select_pairs_kernel<float><<<grid, block, 0, s>>>(
        (const float*)q, (const float*)k, T, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim,
        cfg.r_pairs, pair_idx, contrib);
  return cudaGetLastError();
}
