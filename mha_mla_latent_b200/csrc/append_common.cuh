// Decode-step append shared by the append entry point and the fused decode step:
// c = x W_dkv and the RoPE key dims x W_krope, rotated at the token's position, stored in
// the cache encoding (bf16, or int4/int2 codes with fp16 group scales, plus the residual
// window ring).
//
// Paper notes "MHA2MLA" (ACL 2025), §关键设计: SVDjoint gives the down-projection
// W_dkv whose output c_kv is cached; partial-RoPE keeps each head's selected pairs,
// rotated at the token's position; §与 KV Cache 量化兼容: quantisation of c_kv.
#pragma once

#include "common.cuh"
#include "sm100.cuh"
#include "warp_mma.cuh"

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
  // fused decode step: token n goes to sequence n at position step_lens[n] - 1 (seq_idx
  // and pos unused), and the residual ring slots are claimed inline (one token per
  // sequence, so no two tokens of a call compete for a slot)
  const int32_t* step_lens;
};

// Slot of token n: (sequence, position) from the call's arrays, or for the fused decode
// step from the sequence lengths.  Caller inputs: read only after the dependency wait.
__device__ __forceinline__ void append_slot(const AppendArgs& a, int n, int* sq, int* p) {
  if (n >= a.N) { *sq = -1; *p = -1; return; }
  if (a.step_lens) { *sq = n; *p = __ldg(a.step_lens + n) - 1; return; }
  *sq = __ldg(a.seq_idx + n);
  *p = __ldg(a.pos + n);
}

// Residual window (MLA_CACHE_INT4_G32_R128): the unquantised latent of token (sq, p), in
// the config dtype (bf16), goes to ring slot p % 128 when the slot is claimed by p: by the
// claim kernel that ran first (which left there the largest position of the call for the
// slot), or, in the fused decode step, by the atomic maximum the writer takes itself
// (`claim`; every writer of the row takes it, so they all agree).
__device__ __forceinline__ bool resid_owns(const mla_cache_t& c, int sq, int p, bool claim) {
  if (!c.c_resid) return false;
  int32_t* rp = c.resid_pos + (size_t)sq * MLA_RESID_WINDOW + (p & (MLA_RESID_WINDOW - 1));
  return claim ? atomicMax(rp, p) <= p : *rp == p;
}
__device__ __forceinline__ void resid_store(const mla_cache_t& c, int sq, int p, int d_c, int col, float v) {
  const size_t rs = (size_t)sq * MLA_RESID_WINDOW + (p & (MLA_RESID_WINDOW - 1));
  ((__nv_bfloat16*)c.c_resid)[rs * d_c + col] = __float2bfloat16_rn(v);
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
  // the scratch and the cache may still be in use by the kernels before this one (a
  // second wait, after the one before the caller's inputs, returns at once)
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
      float sn, cs;
      rope_sincos(p, s_theta[cp], &sn, &cs);
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
      const bool own = __shfl_sync(0xffffffffu, lane == 0 ? resid_owns(c, sq, p, a.step_lens != nullptr) : false, 0);
      if (own) resid_store(c, sq, p, a.d_c, col0 + lane, v);
    }
  }
}

// bf16 form of the decode-step append: the slice product runs on the tensor cores as
// m16n8k16 warp MMAs from bf16 tiles staged with cp.async (x [32][ks], W [ks][32], rows
// padded by 16 bytes so the ldmatrix reads are conflict-free); warp w takes hidden dims
// [w ks/8, (w+1) ks/8) for the whole 32 x 32 tile.
//
// (bx, by, bz) is the CTA's (column tile, token tile, hidden-dim slice) in a grid of
// gx x gy x kAppSplit; `sm8` is its dynamic shared memory.  The slice of W_app is staged
// before the dependency wait (plan weights); the caller's x, seq_idx/pos (or sequence
// lengths) only after it.
template <bool INT4>
__device__ __forceinline__ void append_small_mma_body(const AppendSmallArgs& sa, int bx, int by, int bz, int gx,
                                                      int gy, uint8_t* sm8) {
  using bf16 = __nv_bfloat16;
  const AppendArgs& a = sa.a;
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
  const int col0 = bx * kSmCols, tok0 = by * kSmTok;
  const int split = bz;
  const int tile = by * gx + bx, ntile = gx * gy;
  const int k_begin = split * ks, k_end = min(a.d, k_begin + ks);
  const bf16* x = (const bf16*)a.x;
  const bf16* W = (const bf16*)a.W;
  if (tid >= kSmTok && tid < kSmTok + kSmCols / 2) {
    const int cp = tid - kSmTok, col = col0 + 2 * cp;
    double th = 0.0;
    if (col >= a.d_c && col < a.ncols) {
      const int rc = col - a.d_c, g = rc / (2 * a.r), j = (rc % (2 * a.r)) / 2;
      th = __ldg(a.theta + __ldg(a.rope_pair + g * a.r + j));
    }
    s_theta[cp] = th;
  }
  // ---- stage: 16-byte asynchronous copies, all in flight together (missing rows and
  // columns are zero-filled): the weight slice first, the caller's tokens after the wait
  {
    const int nwv = ks * (kSmCols / 8);
    for (int vw = tid; vw < nwv; vw += 256) {
      const int kk = vw / (kSmCols / 8), part = vw % (kSmCols / 8);
      const int kd = k_begin + kk, col = col0 + part * 8;
      const bool ok = kd < k_end && col + 8 <= a.ncols;
      sm100::cp_async16(wmma16::smem_addr(wsm + kk * WLD + part * 8),
                        ok ? (const void*)(W + (size_t)kd * a.ncols + col) : a.W, ok ? 16u : 0u);
    }
    sm100::cp_async_commit();
  }
  pdl_wait();
  pdl_trigger();
  if (tid < kSmTok) append_slot(a, tok0 + tid, &s_sq[tid], &s_pos[tid]);
  {
    const int nxv = kSmTok * (ks / 8);
    for (int v = tid; v < nxv; v += 256) {
      const int t = v / (ks / 8), ch = v % (ks / 8);
      const int n = tok0 + t, kd = k_begin + ch * 8;
      const bool ok = n < a.N && kd + 8 <= k_end;
      sm100::cp_async16(wmma16::smem_addr(xs + t * XLD + ch * 8), ok ? (const void*)(x + (size_t)n * a.d + kd) : a.x,
                        ok ? 16u : 0u);
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

}  // namespace mla

// The fused decode step's append (token b to sequence b at position seq_lens[b] - 1) in its
// bf16 tensor-core form: false when the shape or dtype does not allow that form.
bool mla_append_step_mma_form(const mla_plan& p, const void* x, const int32_t* seq_lens, int B,
                              const mla_cache_t& c, mla::AppendSmallArgs* sa, dim3* grid, size_t* smem);
