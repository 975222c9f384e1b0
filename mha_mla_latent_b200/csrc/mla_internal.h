// Internal declarations shared by the host API (mla_api.cpp) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "mla_api.h"

// Element offset of RoPE key dim j of KV head g, token t of sequence b, in the token-major
// k_rope layout [B][T_cap][n_kv][2r] (one row of n_kv*2r values per token, like c_kv).
inline __host__ __device__ size_t mla_kr_offset(int b, int t, int g, int j, int T_cap, int n_kv, int r2) {
  return (((size_t)b * T_cap + (size_t)t) * n_kv + g) * r2 + j;
}

// Storage location of token t of sequence b: (row-space sequence pb, token pt, capacity cap).
// Contiguous cache: (b, t, T_cap).  Paged cache: (block_table[b][t/128], t % 128, 128), the
// block id checked against the pool (outside it: error flag, block 0).  A token row index
// is pb * cap + pt; RoPE keys sit at mla_kr_offset(pb, pt, g, j, cap, n_kv, 2r).
struct MlaLoc {
  int pb, pt, cap;
};
#ifdef __CUDACC__
inline __device__ MlaLoc mla_loc(const mla_cache_t& c, int b, int t, int32_t* err) {
  if (!c.block_table) return MlaLoc{b, t, c.T_cap};
  int blk = __ldg(c.block_table + (size_t)b * (c.T_cap / MLA_BLOCK_TOKENS) + t / MLA_BLOCK_TOKENS);
  if (blk < 0 || blk >= c.n_blocks) {
    atomicOr(err, MLA_DEVERR_BLOCK);
    blk = 0;
  }
  return MlaLoc{blk, t & (MLA_BLOCK_TOKENS - 1), MLA_BLOCK_TOKENS};
}
#endif
// Token rows in the arrays of the cache (the pool's rows when paged).
inline __host__ __device__ size_t mla_cache_rows(const mla_cache_t& c) {
  return c.block_table ? (size_t)c.n_blocks * MLA_BLOCK_TOKENS : (size_t)c.B * c.T_cap;
}

// True for the int4 cache encodings (with or without the residual window).
inline __host__ __device__ bool mla_kind_int4(int kind) {
  return kind == MLA_CACHE_INT4_G32 || kind == MLA_CACHE_INT4_G32_R128;
}

inline __host__ __device__ bool mla_kind_int2(int kind) { return kind == MLA_CACHE_INT2_G32; }
// Quantised latent (codes + fp16 group scales), and the code width in bits.
inline __host__ __device__ bool mla_kind_quant(int kind) { return mla_kind_int4(kind) || mla_kind_int2(kind); }
inline __host__ __device__ int mla_quant_bits(int kind) { return mla_kind_int2(kind) ? 2 : 4; }

// Host validation of a cache view against a config (mla_api.cpp); MLA_OK when usable.
mla_status_t mla_validate_cache(const mla_config_t& cfg, const mla_cache_t* c);

// Largest token count the decode-step append path takes (its scratch is sized for it).
constexpr int kAppMaxSmallTokens = 128;

struct mla_plan {
  mla_config_t cfg;
  int device = 0;
  int num_sms = 0;
  int R = 0;       // n_kv * 2r   (RoPE key dims per token)
  int dn = 0;      // d_h - 2r    (NoPE dims per head)
  int ncols = 0;   // d_c + R     (columns of the packed append weight)
  // plan-owned device memory
  void* W_app = nullptr;       // [d][ncols] dtype: [W_dkv | W_krope]
  void* W_ukF = nullptr;       // [n_kv][d_h][d_c] dtype: W_uk^T on the NoPE dims, zero rows on the kept pairs
  void* W_uv = nullptr;        // [n_kv][d_c][d_h] dtype
  int32_t* rope_pair = nullptr;  // [n_kv][r]   kept pair indices, ascending
  double* theta = nullptr;       // [d_h/2]     RoPE frequencies
  int32_t* err = nullptr;        // device error word (MLA_DEVERR_* bits)
  float* app_part = nullptr;     // decode-step append: partial tiles [8][tiles][32*32]
  int32_t* app_ticket = nullptr; // decode-step append: per-tile arrival counters (zeroed)
  // options
  int opt_kernel = 0;
  int opt_splits = 0;
  const void* const* opt_events = nullptr;  // cudaEvent_t[2] or null
  const void* const* opt_kernel_events = nullptr;  // cudaEvent_t[8] or null
  int opt_pdl = 1;                            // programmatic dependent launch
  int64_t opt_wait_us = 1000000;              // bound of each pipeline wait (tensor-core kernel)
  int opt_skip_tile = 0;                      // testing: leave out one latent copy per CTA
};

// Launches a kernel, with programmatic stream serialization when `pdl` is set (the kernel
// then orders itself after its predecessor with griddepcontrol.wait).
template <typename... KArgs, typename... Args>
inline cudaError_t mla_launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                     bool pdl, Args&&... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&lc, kern, std::forward<Args>(args)...);
}

// Kernels of a call that the profiling options can bracket with events.
enum MlaProfKernel { kProfAppend = 0, kProfAbsorb = 1, kProfAttention = 2, kProfCombine = 3 };

// Records the profiling event before (`after` false) or after a kernel launch when an
// option asks for it: MLA_OPT_PROFILE_EVENTS brackets the split-K attention kernel,
// MLA_OPT_PROFILE_KERNELS every kernel.  Under stream capture the record becomes an
// external event node of the graph, so the event still marks each replay.  A failed record
// is returned, never left pending.
inline cudaError_t mla_profile_event(const mla_plan& p, MlaProfKernel k, bool after, cudaStream_t s) {
  const void* ev = nullptr;
  if (p.opt_kernel_events) ev = p.opt_kernel_events[2 * (int)k + (after ? 1 : 0)];
  else if (p.opt_events && k == kProfAttention) ev = p.opt_events[after ? 1 : 0];
  if (!ev) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  return cudaEventRecordWithFlags((cudaEvent_t)ev, s,
                                  cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                                      : cudaEventRecordDefault);
}

// Decode workspace layout (byte offsets from the workspace base).
struct DecodeLayout {
  int kernel = 1;          // 1 CUDA-core, 2 tcgen05 decode (token rows), 3 tcgen05 query
                           // chunks, 4 tcgen05 decode (head rows: the chunk kernel's form)
  int tile = 32;           // tokens per schedule tile
  int G = 0;               // workers (CTAs of the split-K kernel)
  int P = 0;               // max pieces = B + G
  int K = 0;               // tcgen05 query row width (d_c + R)
  size_t off_seq_tile0, off_seq_ntiles, off_seq_ne, off_seq_first, off_seq_np;
  size_t off_worker_first, off_piece_b, off_piece_t0, off_piece_t1;
  size_t off_qlat, off_qrope, off_opart, off_mlpart;
  size_t total = 0;
};

// Schedule view passed to kernels (pointers into the workspace).
struct Sched {
  int32_t* seq_tile0;     // [B]  first global tile of sequence b
  int32_t* seq_ntiles;    // [B]
  int32_t* seq_ne;        // [B+1] number of non-empty sequences before b
  int32_t* seq_first;     // [B]  first piece of b
  int32_t* seq_np;        // [B]  pieces of b
  int32_t* worker_first;  // [G+1]
  int32_t* piece_b;       // [P]
  int32_t* piece_t0;      // [P] token begin within sequence
  int32_t* piece_t1;      // [P] token end (exclusive)
};

DecodeLayout mla_decode_layout(const mla_plan& p, int B, int kernel);
bool mla_tc_supported(const mla_plan& p, const mla_cache_t& c);
bool mla_tc_capable(const mla_plan& p);   // shape/dtype allow the tensor-core kernel
cudaError_t mla_launch_decode_tc(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, int B,
                                 const Sched& sched,
                                 const void* qlat, const float* qrope, float* opart, float* mlpart, int P, int G,
                                 cudaStream_t s);
Sched mla_sched_view(const DecodeLayout& L, void* ws, int B);
// Many queries per sequence: workspace layout, the chunk kernel's shape limits and launches.
DecodeLayout mla_chunk_layout(const mla_plan& p, int B, int Q);
bool mla_chunk_capable(const mla_plan& p);
bool mla_chunk_supported(const mla_plan& p, const mla_cache_t& c);
// rows = 128: units of floor(128 / H) queries x H heads (query chunks, and decode with more
// than 32 heads); rows = 32: one query's heads (decode with up to 32 heads)
cudaError_t mla_launch_chunk_tc(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, int B, int Q,
                                const Sched& sched, const void* qlat, const float* qrope, float* opart,
                                float* mlpart, int P, int G, cudaStream_t s, int rows);
bool mla_decode_t_capable(const mla_plan& p);
bool mla_decode_t_supported(const mla_plan& p, const mla_cache_t& c);
// The decode kernel a call runs (layout kernel id 1, 2 or 4), or the status refusing the call.
mla_status_t mla_pick_decode_kernel(const mla_plan& p, const mla_cache_t& c, int* kernel);
cudaError_t mla_launch_chunk(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, const void* q,
                             int B, int Q, void* out, void* ws, const DecodeLayout& L, cudaStream_t s);

cudaError_t mla_launch_select_pairs(const mla_config_t& cfg, const void* q, const void* k, int T,
                                    int32_t* pair_idx, float* contrib, cudaStream_t s);
cudaError_t mla_launch_append(const mla_plan& p, const void* x, const int32_t* seq_idx,
                              const int32_t* pos, int N, const mla_cache_t& c, cudaStream_t s);
// Append of a decode step: token b goes to sequence b at position seq_lens[b] - 1.
cudaError_t mla_launch_append_step(const mla_plan& p, const void* x, const int32_t* seq_lens, int B,
                                   const mla_cache_t& c, cudaStream_t s);
// One decode step (append of each sequence's new token, then decode), fused where it can be.
cudaError_t mla_launch_step(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, const void* x,
                            const void* q, int B, void* out, void* ws, const DecodeLayout& L, cudaStream_t s);
cudaError_t mla_launch_decode(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens,
                              const void* q, int B, void* out, void* ws, const DecodeLayout& L,
                              cudaStream_t s);
