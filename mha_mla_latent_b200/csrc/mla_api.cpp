// Host side of the C ABI: argument validation, plan construction (weight packing),
// workspace layout and kernel launches.  See include/mla_api.h for the contract.
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include "mla_internal.h"

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

size_t elem_bytes(const mla_config_t& c) { return c.dtype == MLA_F32 ? 4 : 2; }

mla_status_t validate_config(const mla_config_t* c) {
  if (!c) return MLA_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 || c->d_c <= 0)
    return MLA_ERR_INVALID_ARG;
  if (c->n_heads % c->n_kv_heads != 0 || c->head_dim % 2 != 0) return MLA_ERR_INVALID_ARG;
  if (c->r_pairs < 0 || 2 * c->r_pairs > c->head_dim) return MLA_ERR_INVALID_ARG;
  if (!(c->rope_base > 1.0)) return MLA_ERR_INVALID_ARG;
  if (!(c->softmax_scale >= 0.0f) || !isfinite(c->softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (c->dtype != MLA_F32 && c->dtype != MLA_BF16) return MLA_ERR_INVALID_ARG;
  if (c->cache_kind != MLA_CACHE_SAME && !mla_kind_quant(c->cache_kind)) return MLA_ERR_INVALID_ARG;
  if (mla_kind_quant(c->cache_kind) && (c->dtype != MLA_BF16 || c->d_c % 32 != 0))
    return MLA_ERR_UNSUPPORTED;
  // limits of the kernels in this build
  if (c->head_dim > 256 || c->d_c > 1024 || c->n_heads > 256) return MLA_ERR_UNSUPPORTED;
  if (c->d_c % 4 != 0) return MLA_ERR_UNSUPPORTED;   // float4 rows in the split merge
  return MLA_OK;
}

}  // namespace

mla_status_t mla_validate_cache(const mla_config_t& cfg, const mla_cache_t* c) {
  if (!c || !c->c_kv || c->B <= 0 || c->T_cap <= 0) return MLA_ERR_INVALID_ARG;
  const bool quant = mla_kind_quant(cfg.cache_kind);
  if (quant != (c->c_scales != nullptr)) return MLA_ERR_INVALID_ARG;
  if (cfg.r_pairs > 0 && !c->k_rope) return MLA_ERR_INVALID_ARG;
  if (c->block_table) {   // paged: 128-token blocks, a table row per sequence
    if (c->n_blocks <= 0 || c->T_cap % MLA_BLOCK_TOKENS != 0) return MLA_ERR_INVALID_ARG;
    if ((uintptr_t)c->block_table % 4 != 0) return MLA_ERR_ALIGNMENT;
  } else if (c->n_blocks != 0) {
    return MLA_ERR_INVALID_ARG;
  }
  // The attention kernels name a token row by a signed 32-bit TMA coordinate.
  if (mla_cache_rows(*c) > (size_t)INT32_MAX) return MLA_ERR_UNSUPPORTED;
  const bool resid = cfg.cache_kind == MLA_CACHE_INT4_G32_R128;
  if (resid != (c->c_resid != nullptr) || resid != (c->resid_pos != nullptr)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(c->c_kv) || (c->c_scales && !aligned16(c->c_scales)) ||
      (c->k_rope && !aligned16(c->k_rope)) || (c->c_resid && !aligned16(c->c_resid)) ||
      (c->resid_pos && !aligned16(c->resid_pos)))
    return MLA_ERR_ALIGNMENT;
  return MLA_OK;
}

namespace {

mla_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

bool dev_alloc_copy(void** dst, const void* src, size_t bytes) {
  if (cudaMalloc(dst, bytes) != cudaSuccess) { *dst = nullptr; return false; }
  return cudaMemcpy(*dst, src, bytes, cudaMemcpyHostToDevice) == cudaSuccess;
}

void free_plan(mla_plan* p) {
  if (!p) return;
  void* bufs[] = {p->W_app, p->W_ukF, p->W_uv, p->rope_pair, p->theta, p->err, p->app_part, p->app_ticket};
  for (void* b : bufs)
    if (b) cudaFree(b);
  delete p;
}

}  // namespace

// The decode kernel a call runs: the tensor-core kernel where the plan, cache and options
// allow it, else the CUDA-core kernel.  MLA_OK, or the status that refuses the call.
// Kernel ids of the decode layout: 1 CUDA cores, 2 tcgen05 token rows, 4 tcgen05 head rows.
mla_status_t mla_pick_decode_kernel(const mla_plan& p, const mla_cache_t& c, int* kernel) {
  *kernel = 1;
  const bool head_rows = mla_decode_t_supported(p, c);
  const bool token_rows = mla_tc_supported(p, c);
  switch (p.opt_kernel) {
    case 1: break;
    case 2:
      if (!token_rows) return MLA_ERR_UNSUPPORTED;
      *kernel = 2;
      break;
    case 3:
      if (!head_rows) return MLA_ERR_UNSUPPORTED;
      *kernel = 4;
      break;
    default:   // the head-row kernel where its shapes allow, else the token-row kernel
      if (head_rows) *kernel = 4;
      else if (token_rows) *kernel = 2;
      break;
  }
  if (*kernel == 1 && (size_t)p.cfg.n_heads * p.cfg.d_c > 8192) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

extern "C" {

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MLA_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_DEVICE: return "device-side error recorded";
  }
  return "unknown status";
}

const char* mla_version(void) { return "mla_b200 0.1 (sm_100a)"; }

size_t mla_cache_bytes_per_token(const mla_config_t* cfg) {
  if (validate_config(cfg) == MLA_ERR_INVALID_ARG) return 0;
  size_t eb = elem_bytes(*cfg);
  size_t rope = (size_t)cfg->n_kv_heads * 2 * cfg->r_pairs * eb;
  if (mla_kind_int4(cfg->cache_kind)) return (size_t)cfg->d_c / 2 + 2 * ((size_t)cfg->d_c / 32) + rope;
  if (mla_kind_int2(cfg->cache_kind)) return (size_t)cfg->d_c / 4 + 2 * ((size_t)cfg->d_c / 32) + rope;
  return (size_t)cfg->d_c * eb + rope;
}

mla_status_t mla_fixed_pairs(const mla_config_t* cfg, int32_t strategy, int32_t* pair_idx) {
  if (!cfg || !pair_idx) return MLA_ERR_INVALID_ARG;
  mla_status_t st = validate_config(cfg);
  if (st != MLA_OK) return st;
  const int P = cfg->head_dim / 2, r = cfg->r_pairs, nkv = cfg->n_kv_heads;
  if (r < 0 || r > P) return MLA_ERR_INVALID_ARG;
  std::vector<int32_t> ks(r);
  switch (strategy) {
    case MLA_PAIRS_HIGH:
      for (int j = 0; j < r; ++j) ks[j] = j;
      break;
    case MLA_PAIRS_LOW:
      for (int j = 0; j < r; ++j) ks[j] = P - r + j;
      break;
    case MLA_PAIRS_UNIFORM:
      for (int j = 0; j < r; ++j) ks[j] = (int32_t)(((long long)j * P) / r);
      break;
    case MLA_PAIRS_FULL:
      if (r != P) return MLA_ERR_INVALID_ARG;
      for (int j = 0; j < r; ++j) ks[j] = j;
      break;
    default:
      return MLA_ERR_INVALID_ARG;
  }
  for (int g = 0; g < nkv; ++g)
    for (int j = 0; j < r; ++j) pair_idx[(size_t)g * r + j] = ks[j];
  return MLA_OK;
}

mla_status_t mla_select_pairs(const mla_config_t* cfg, const void* q_cal, const void* k_cal,
                              int32_t T, int32_t* pair_idx, float* contrib, void* stream) {
  mla_status_t st = validate_config(cfg);
  if (st != MLA_OK) return st;
  if (!q_cal || !k_cal || !pair_idx || T <= 0) return MLA_ERR_INVALID_ARG;
  if (cfg->head_dim / 2 > 128) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(q_cal) || !aligned16(k_cal)) return MLA_ERR_ALIGNMENT;
  return cuda_status(mla_launch_select_pairs(*cfg, q_cal, k_cal, T, pair_idx, contrib,
                                             (cudaStream_t)stream));
}

namespace {

// Packs the converted weights on the host and copies them into plan-owned device memory:
// [W_dkv | W_krope], W_uk spread over the full head dims, W_uv, the pair tables, the
// frequencies and the append scratch.  False when a device allocation or copy fails; host
// allocation failures throw std::bad_alloc, which mla_plan_create turns into a status.
bool pack_and_upload(mla_plan* p, const void* W_dkv, const void* W_k, const int32_t* pair_idx, const void* W_uk,
                     const void* W_uv) {
  const int d = p->cfg.hidden, nkv = p->cfg.n_kv_heads, dh = p->cfg.head_dim, r = p->cfg.r_pairs;
  const int dc = p->cfg.d_c;
  const size_t eb = elem_bytes(p->cfg);
  // [W_dkv | W_krope]: column block of the selected pairs of each KV head, ascending.
  std::vector<unsigned char> app((size_t)d * p->ncols * eb);
  for (int i = 0; i < d; ++i) {
    memcpy(&app[((size_t)i * p->ncols) * eb], (const unsigned char*)W_dkv + (size_t)i * dc * eb, dc * eb);
    for (int g = 0; g < nkv; ++g)
      for (int j = 0; j < r; ++j)
        for (int e = 0; e < 2; ++e) {
          int src_col = g * dh + 2 * pair_idx[g * r + j] + e;
          int dst_col = dc + g * 2 * r + 2 * j + e;
          memcpy(&app[((size_t)i * p->ncols + dst_col) * eb],
                 (const unsigned char*)W_k + ((size_t)i * nkv * dh + src_col) * eb, eb);
        }
  }
  // W_uk transposed per head onto the full head dims: [g][d][c] = W_uk[g][c][j] where d is
  // the j-th NoPE dim of KV head g; the rows of the kept pairs' dims stay zero, so an
  // unrotated query can be multiplied as it is
  std::vector<unsigned char> ukF((size_t)nkv * dh * dc * eb, 0);
  std::vector<int32_t> rp((size_t)nkv * std::max(r, 1), 0);
  for (int g = 0; g < nkv; ++g) {
    std::vector<char> kept(dh / 2, 0);
    for (int j = 0; j < r; ++j) { kept[pair_idx[g * r + j]] = 1; rp[g * r + j] = pair_idx[g * r + j]; }
    int j = 0;
    for (int hd = 0; hd < dh; ++hd) {
      if (kept[hd / 2]) continue;
      for (int c = 0; c < dc; ++c)
        memcpy(&ukF[(((size_t)g * dh + hd) * dc + c) * eb],
               (const unsigned char*)W_uk + (((size_t)g * dc + c) * p->dn + j) * eb, eb);
      ++j;
    }
  }
  std::vector<double> theta(dh / 2);
  for (int k = 0; k < dh / 2; ++k) theta[k] = pow(p->cfg.rope_base, -2.0 * k / dh);

  bool ok = dev_alloc_copy(&p->W_app, app.data(), app.size()) &&
            dev_alloc_copy(&p->W_ukF, ukF.data(), ukF.size()) &&
            dev_alloc_copy(&p->W_uv, W_uv, (size_t)nkv * dc * dh * eb) &&
            dev_alloc_copy((void**)&p->rope_pair, rp.data(), rp.size() * sizeof(int32_t)) &&
            dev_alloc_copy((void**)&p->theta, theta.data(), theta.size() * sizeof(double)) &&
            cudaMalloc((void**)&p->err, sizeof(int32_t)) == cudaSuccess &&
            cudaMemset(p->err, 0, sizeof(int32_t)) == cudaSuccess;
  // decode-step append scratch: 8 hidden-dim slices x (tiles of 32 tokens x 32 columns)
  const size_t app_tiles = (size_t)((p->ncols + 31) / 32) * ((kAppMaxSmallTokens + 31) / 32);
  ok = ok && cudaMalloc((void**)&p->app_part, app_tiles * 8 * 32 * 32 * sizeof(float)) == cudaSuccess &&
       cudaMalloc((void**)&p->app_ticket, app_tiles * sizeof(int32_t)) == cudaSuccess &&
       cudaMemset(p->app_ticket, 0, app_tiles * sizeof(int32_t)) == cudaSuccess;
  return ok;
}

}  // namespace

mla_status_t mla_plan_create(const mla_config_t* cfg, const void* W_dkv, const void* W_k,
                             const int32_t* pair_idx, const void* W_uk, const void* W_uv,
                             mla_plan_t** out) {
  if (!out) return MLA_ERR_INVALID_ARG;
  *out = nullptr;
  mla_status_t st = validate_config(cfg);
  if (st != MLA_OK) return st;
  const int nkv = cfg->n_kv_heads, dh = cfg->head_dim, r = cfg->r_pairs;
  if (!W_dkv || !W_uv || (dh - 2 * r > 0 && !W_uk) || (r > 0 && (!W_k || !pair_idx)))
    return MLA_ERR_INVALID_ARG;
  for (int g = 0; g < nkv; ++g)
    for (int j = 0; j < r; ++j) {
      int k = pair_idx[g * r + j];
      if (k < 0 || k >= dh / 2) return MLA_ERR_INVALID_ARG;
      if (j > 0 && k <= pair_idx[g * r + j - 1]) return MLA_ERR_INVALID_ARG;  // strictly ascending
    }
  mla_plan* p = new (std::nothrow) mla_plan();
  if (!p) return MLA_ERR_CUDA;
  p->cfg = *cfg;
  p->R = nkv * 2 * r;
  p->dn = dh - 2 * r;
  p->ncols = cfg->d_c + p->R;
  if (cudaGetDevice(&p->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess) {
    free_plan(p);
    return MLA_ERR_CUDA;
  }
  bool ok = false;
  try {
    ok = pack_and_upload(p, W_dkv, W_k, pair_idx, W_uk, W_uv);
  } catch (const std::exception&) {   // no host memory for the packed copies
    ok = false;
  }
  if (!ok) {
    free_plan(p);
    return MLA_ERR_CUDA;
  }
  *out = p;
  return MLA_OK;
}

void mla_plan_destroy(mla_plan_t* plan) { free_plan(plan); }

mla_status_t mla_plan_set_option(mla_plan_t* plan, int32_t option, int64_t value) {
  if (!plan) return MLA_ERR_INVALID_ARG;
  switch (option) {
    case MLA_OPT_DECODE_KERNEL:
      if (value < 0 || value > 3) return MLA_ERR_INVALID_ARG;
      plan->opt_kernel = (int)value;
      return MLA_OK;
    case MLA_OPT_DECODE_SPLITS:
      if (value < 0 || value > (1 << 20)) return MLA_ERR_INVALID_ARG;
      plan->opt_splits = (int)value;
      return MLA_OK;
    case MLA_OPT_PROFILE_EVENTS:
      plan->opt_events = (const void* const*)(uintptr_t)value;
      return MLA_OK;
    case MLA_OPT_PROFILE_KERNELS:
      plan->opt_kernel_events = (const void* const*)(uintptr_t)value;
      return MLA_OK;
    case MLA_OPT_OVERLAP_LAUNCH:
      if (value < 0 || value > 1) return MLA_ERR_INVALID_ARG;
      plan->opt_pdl = (int)value;
      return MLA_OK;
    case MLA_OPT_WAIT_LIMIT_US:
      if (value < 100 || value > 10000000) return MLA_ERR_INVALID_ARG;
      plan->opt_wait_us = value;
      return MLA_OK;
    case MLA_OPT_TEST_SKIP_COPY:
      if (value < 0 || value > (1 << 20)) return MLA_ERR_INVALID_ARG;
      plan->opt_skip_tile = (int)value;
      return MLA_OK;

  }
  return MLA_ERR_INVALID_ARG;
}

mla_status_t mla_append(const mla_plan_t* plan, const void* x, const int32_t* seq_idx,
                        const int32_t* pos, int32_t N, const mla_cache_t* cache, void* stream) {
  if (!plan || !x || !seq_idx || !pos || N <= 0) return MLA_ERR_INVALID_ARG;
  mla_status_t st = mla_validate_cache(plan->cfg, cache);
  if (st != MLA_OK) return st;
  if (!aligned16(x) || ((uintptr_t)seq_idx & 3) || ((uintptr_t)pos & 3)) return MLA_ERR_ALIGNMENT;
  const cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = mla_profile_event(*plan, kProfAppend, false, s);
  if (e == cudaSuccess) e = mla_launch_append(*plan, x, seq_idx, pos, N, *cache, s);
  if (e == cudaSuccess) e = mla_profile_event(*plan, kProfAppend, true, s);
  return cuda_status(e);
}

namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Staging of mla_decode_step_host inside the workspace, after the decode's own part:
// seq_lens, x, q and out, each 256-byte aligned.
struct HostStage {
  size_t off_lens, off_x, off_q, off_out, total;
};
HostStage host_stage(const mla_plan& p, int B, size_t base) {
  const mla_config_t& c = p.cfg;
  const size_t eb = elem_bytes(c), qo = (size_t)B * c.n_heads * c.head_dim * eb;
  HostStage h;
  h.off_lens = align256(base);
  h.off_x = h.off_lens + align256((size_t)B * sizeof(int32_t));
  h.off_q = h.off_x + align256((size_t)B * c.hidden * eb);
  h.off_out = h.off_q + align256(qo);
  h.total = h.off_out + align256(qo);
  return h;
}

mla_status_t pick_kernel(const mla_plan& p, const mla_cache_t& c, int* kernel) {
  return mla_pick_decode_kernel(p, c, kernel);
}

}  // namespace

mla_status_t mla_decode_kernel_choice(const mla_plan_t* plan, const mla_cache_t* cache, int32_t* kernel) {
  if (!plan || !cache || !kernel) return MLA_ERR_INVALID_ARG;
  int k = 1;
  const mla_status_t st = mla_pick_decode_kernel(*plan, *cache, &k);
  if (st != MLA_OK) return st;
  *kernel = k == 4 ? 3 : k;
  return MLA_OK;
}

size_t mla_decode_workspace_bytes(const mla_plan_t* plan, int32_t B) {
  if (!plan || B <= 0) return 0;
  size_t n = mla_decode_layout(*plan, B, 1).total;
  if (mla_tc_capable(*plan)) n = std::max(n, mla_decode_layout(*plan, B, 2).total);
  if (mla_decode_t_capable(*plan)) n = std::max(n, mla_decode_layout(*plan, B, 4).total);
  return host_stage(*plan, B, n).total;
}

mla_status_t mla_decode(const mla_plan_t* plan, const mla_cache_t* cache, const int32_t* seq_lens,
                        const void* q, int32_t B, void* out, void* workspace, size_t ws_bytes,
                        void* stream) {
  if (!plan || !seq_lens || !q || !out || !workspace || B <= 0) return MLA_ERR_INVALID_ARG;
  mla_status_t st = mla_validate_cache(plan->cfg, cache);
  if (st != MLA_OK) return st;
  if (B > cache->B) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace) || ((uintptr_t)seq_lens & 3))
    return MLA_ERR_ALIGNMENT;
  int kernel = 1;
  if ((st = pick_kernel(*plan, *cache, &kernel)) != MLA_OK) return st;
  DecodeLayout L = mla_decode_layout(*plan, B, kernel);
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  return cuda_status(mla_launch_decode(*plan, *cache, seq_lens, q, B, out, workspace, L,
                                       (cudaStream_t)stream));
}

size_t mla_decode_chunk_workspace_bytes(const mla_plan_t* plan, int32_t B, int32_t Q) {
  if (!plan || B <= 0 || Q <= 0) return 0;
  if (Q == 1) return mla_decode_workspace_bytes(plan, B);
  return mla_chunk_layout(*plan, B, Q).total;
}

mla_status_t mla_decode_chunk(const mla_plan_t* plan, const mla_cache_t* cache, const int32_t* seq_lens,
                              const void* q, int32_t B, int32_t Q, void* out, void* workspace, size_t ws_bytes,
                              void* stream) {
  if (!plan || !seq_lens || !q || !out || !workspace || B <= 0 || Q <= 0) return MLA_ERR_INVALID_ARG;
  if (Q == 1) return mla_decode(plan, cache, seq_lens, q, B, out, workspace, ws_bytes, stream);
  mla_status_t st = mla_validate_cache(plan->cfg, cache);
  if (st != MLA_OK) return st;
  if (B > cache->B || (long long)Q > cache->T_cap) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace) || ((uintptr_t)seq_lens & 3))
    return MLA_ERR_ALIGNMENT;
  if (!mla_chunk_supported(*plan, *cache) || plan->opt_kernel == 1) return MLA_ERR_UNSUPPORTED;
  DecodeLayout L = mla_chunk_layout(*plan, B, Q);
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  return cuda_status(mla_launch_chunk(*plan, *cache, seq_lens, q, B, Q, out, workspace, L, (cudaStream_t)stream));
}

mla_status_t mla_decode_step(const mla_plan_t* plan, const mla_cache_t* cache, const int32_t* seq_lens,
                             const void* x, const void* q, int32_t B, void* out, void* workspace, size_t ws_bytes,
                             void* stream) {
  if (!plan || !seq_lens || !x || !q || !out || !workspace || B <= 0) return MLA_ERR_INVALID_ARG;
  mla_status_t st = mla_validate_cache(plan->cfg, cache);
  if (st != MLA_OK) return st;
  if (B > cache->B) return MLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q) || !aligned16(out) || !aligned16(workspace) || ((uintptr_t)seq_lens & 3))
    return MLA_ERR_ALIGNMENT;
  int kernel = 1;
  if ((st = pick_kernel(*plan, *cache, &kernel)) != MLA_OK) return st;
  DecodeLayout L = mla_decode_layout(*plan, B, kernel);
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  return cuda_status(mla_launch_step(*plan, *cache, seq_lens, x, q, B, out, workspace, L, (cudaStream_t)stream));
}

mla_status_t mla_decode_step_host(const mla_plan_t* plan, const mla_cache_t* cache, const int32_t* seq_lens,
                                  const void* x, const void* q, int32_t B, void* out, void* workspace,
                                  size_t ws_bytes, void* stream) {
  if (!plan || !seq_lens || !x || !q || !out || !workspace || B <= 0) return MLA_ERR_INVALID_ARG;
  mla_status_t st = mla_validate_cache(plan->cfg, cache);
  if (st != MLA_OK) return st;
  if (B > cache->B) return MLA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return MLA_ERR_ALIGNMENT;
  int kernel = 1;
  if ((st = pick_kernel(*plan, *cache, &kernel)) != MLA_OK) return st;
  DecodeLayout L = mla_decode_layout(*plan, B, kernel);
  const HostStage h = host_stage(*plan, B, L.total);
  if (ws_bytes < h.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  const mla_config_t& c = plan->cfg;
  const size_t eb = elem_bytes(c), qo = (size_t)B * c.n_heads * c.head_dim * eb;
  char* w = (char*)workspace;
  const cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(w + h.off_lens, seq_lens, (size_t)B * sizeof(int32_t), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(w + h.off_x, x, (size_t)B * c.hidden * eb, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(w + h.off_q, q, qo, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = mla_launch_step(*plan, *cache, (const int32_t*)(w + h.off_lens), w + h.off_x, w + h.off_q, B, w + h.off_out,
                        workspace, L, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(out, w + h.off_out, qo, cudaMemcpyDeviceToHost, s);
  return cuda_status(e);
}

mla_status_t mla_device_error(mla_plan_t* plan, int32_t* code) {
  if (!plan || !code) return MLA_ERR_INVALID_ARG;
  *code = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpy(code, plan->err, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (cudaMemset(plan->err, 0, sizeof(int32_t)) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

}  // extern "C"
