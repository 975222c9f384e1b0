// Decode over the latent cache: query absorption, split-K attention (CUDA-core kernel),
// split merge with W_uv, and the host-side orchestration of one decode step.
//
// Paper notes "MHA2MLA" (ACL 2025), §关键设计: the NoPE key is K_nope = c_kv W_uk and
// the value V = c_kv W_uv (SVDjoint); the RoPE part cannot be merged into the matrices
// and is scored separately.  Absorbing W_uk into the query (q_lat = q_nope W_uk^T)
// scores the NoPE part directly against c_kv; the probability-weighted latent is taken
// through W_uv after the softmax sum.  Scores are kept in log2 units (the query is
// pre-scaled by log2(e)/sqrt(d_h)) so the softmax uses exp2.
#include "decode_common.cuh"

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
};

constexpr int kAbsMaxRows = 16;   // (b, h) rows per CTA

template <typename T>
__global__ void __launch_bounds__(256) absorb_kernel(AbsorbArgs a) {
  const int nchunks = (a.B + a.bchunk - 1) / a.bchunk;
  if (blockIdx.x == a.n_kv * nchunks) {  // the last CTA builds the split-K schedule
    build_schedule(a.seq_lens, a.B, a.T_cap, a.tile, a.G, a.sched, a.err);
    return;
  }
  const int g = blockIdx.x % a.n_kv, chunk = blockIdx.x / a.n_kv;
  const int G = a.H / a.n_kv;
  const int b0 = chunk * a.bchunk;
  const int nb = min(a.bchunk, a.B - b0);
  const int rows = nb * G;
  extern __shared__ float sm[];
  float* qn = sm;                           // [rows][dn]
  const float scale = kLog2e * rsqrtf((float)a.dh);
  const T* q = (const T*)a.q;
  for (int i = threadIdx.x; i < rows * a.dn; i += blockDim.x) {
    int row = i / a.dn, j = i % a.dn;
    int b = b0 + row / G, h = g * G + row % G;
    qn[i] = to_f32(q[((size_t)b * a.H + h) * a.dh + a.nope_idx[g * a.dn + j]]);
  }
  // RoPE part: rotate the kept pairs at position L-1 (angle in double), scale.
  for (int i = threadIdx.x; i < rows * a.r; i += blockDim.x) {
    int row = i / a.r, j = i % a.r;
    int b = b0 + row / G, h = g * G + row % G;
    int L = a.seq_lens[b];
    int p = (L >= 1 && L <= a.T_cap) ? L - 1 : 0;
    int k = a.rope_pair[g * a.r + j];
    const T* qp = q + ((size_t)b * a.H + h) * a.dh + 2 * k;
    double x0 = to_f32(qp[0]), x1 = to_f32(qp[1]);
    double sn, cs;
    sincos((double)p * a.theta[k], &sn, &cs);
    float o0 = (float)((x0 * cs - x1 * sn) * (double)scale);
    float o1 = (float)((x0 * sn + x1 * cs) * (double)scale);
    size_t bh = (size_t)b * a.H + h;
    if (a.qrope) { a.qrope[bh * 2 * a.r + 2 * j] = o0; a.qrope[bh * 2 * a.r + 2 * j + 1] = o1; }
    if (a.qcat) {
      a.qcat[bh * a.K + a.d_c + g * 2 * a.r + 2 * j] = __float2bfloat16_rn(o0);
      a.qcat[bh * a.K + a.d_c + g * 2 * a.r + 2 * j + 1] = __float2bfloat16_rn(o1);
    }
  }
  if (a.qcat) {  // zero the other KV heads' RoPE slots of the concatenated query row
    for (int i = threadIdx.x; i < rows * a.R; i += blockDim.x) {
      int row = i / a.R, j = i % a.R;
      if (j / (2 * a.r) == g) continue;
      size_t bh = (size_t)(b0 + row / G) * a.H + g * G + row % G;
      a.qcat[bh * a.K + a.d_c + j] = __float2bfloat16_rn(0.f);
    }
  }
  __syncthreads();
  // Latent part: q_lat[row][c] = scale * sum_j qn[row][j] * W_uk[g][c][j].
  const T* W = (const T*)a.W_ukT + (size_t)g * a.dn * a.d_c;
  for (int c = threadIdx.x; c < a.d_c; c += blockDim.x) {
    float acc[kAbsMaxRows];
#pragma unroll
    for (int i = 0; i < kAbsMaxRows; ++i) acc[i] = 0.f;
#pragma unroll 8
    for (int j = 0; j < a.dn; ++j) {
      float w = to_f32(W[(size_t)j * a.d_c + c]);
#pragma unroll
      for (int i = 0; i < kAbsMaxRows; ++i)
        if (i < rows) acc[i] += qn[i * a.dn + j] * w;
    }
#pragma unroll
    for (int i = 0; i < kAbsMaxRows; ++i) {
      if (i >= rows) break;
      size_t bh = (size_t)(b0 + i / G) * a.H + g * G + i % G;
      if (a.qlat) a.qlat[bh * a.d_c + c] = acc[i] * scale;
      if (a.qcat) a.qcat[bh * a.K + c] = __float2bfloat16_rn(acc[i] * scale);
    }
  }
}

// ------------------------------------------------------------ CUDA-core split-K decode
struct DecodeArgs {
  mla_cache_t cache;
  int B, H, n_kv, r, d_c, R;
  const float* qlat;
  const float* qrope;
  float* opart;     // [P][H][d_c]
  float* mlpart;    // [P][H][2]
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
        s_kr[tt * (R + 1) + j] = to_f32(((const T*)a.cache.k_rope)[(slot0 + tt) * R + j]);
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
      if (idx < H * dc) a.opart[(size_t)pc * H * dc + idx] = O[e];
    }
    if (tid < H) {
      a.mlpart[((size_t)pc * H + tid) * 2] = s_m[tid];
      a.mlpart[((size_t)pc * H + tid) * 2 + 1] = s_l[tid];
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
};

template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  const int g = blockIdx.x % a.n_kv, chunk = blockIdx.x / a.n_kv;
  const int G = a.H / a.n_kv;
  const int b0 = chunk * a.bchunk;
  const int nb = min(a.bchunk, a.B - b0);
  const int rows = nb * G;
  extern __shared__ float sm[];
  float* s_o = sm;                    // [rows][d_c]
  float* s_M = s_o + rows * a.d_c;    // [rows] merged running max
  float* s_inv = s_M + rows;          // [rows] 1 / merged sum
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  // per (b, h): M = max_j m_j, 1 / sum_j 2^(m_j - M) l_j   (one warp per row)
  for (int row = warp; row < rows; row += nwarp) {
    const int b = b0 + row / G, h = g * G + row % G;
    const int first = a.sched.seq_first[b], np = a.sched.seq_np[b];
    float M = -INFINITY;
    for (int j = lane; j < np; j += 32) M = fmaxf(M, a.mlpart[((size_t)(first + j) * a.H + h) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
    for (int j = lane; j < np; j += 32) {
      const float* ml = a.mlpart + ((size_t)(first + j) * a.H + h) * 2;
      den += exp2f(ml[0] - M) * ml[1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane == 0) {
      s_M[row] = M;
      s_inv[row] = (np > 0 && den > 0.f) ? 1.f / den : 0.f;
    }
  }
  __syncthreads();
  // merged latent O_lat[row][c]
  for (int i = threadIdx.x; i < rows * a.d_c; i += blockDim.x) {
    const int row = i / a.d_c, c = i % a.d_c;
    const int b = b0 + row / G, h = g * G + row % G;
    const int first = a.sched.seq_first[b], np = a.sched.seq_np[b];
    const float M = s_M[row];
    float num = 0.f;
    for (int j = 0; j < np; ++j) {
      const size_t pj = (size_t)(first + j) * a.H + h;
      num += exp2f(a.mlpart[pj * 2] - M) * a.opart[pj * a.d_c + c];
    }
    s_o[i] = num * s_inv[row];
  }
  __syncthreads();
  // o[row][d] = sum_c O_lat[row][c] W_uv[g][c][d]; each thread owns one d for a set of rows
  const T* W = (const T*)a.W_uv + (size_t)g * a.d_c * a.dh;
  constexpr int kRows = 8;
  for (int i = threadIdx.x; i < a.dh * ((rows + kRows - 1) / kRows); i += blockDim.x) {
    const int d = i % a.dh, r0 = (i / a.dh) * kRows;
    float acc[kRows];
#pragma unroll
    for (int k = 0; k < kRows; ++k) acc[k] = 0.f;
#pragma unroll 8
    for (int c = 0; c < a.d_c; ++c) {
      const float wv = to_f32(W[(size_t)c * a.dh + d]);
#pragma unroll
      for (int k = 0; k < kRows; ++k)
        if (r0 + k < rows) acc[k] += s_o[(r0 + k) * a.d_c + c] * wv;
    }
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
  aa.qrope = L.kernel == 1 ? (float*)(base + L.off_qrope) : nullptr;
  aa.qcat = L.kernel == 2 ? (__nv_bfloat16*)(base + L.off_qlat) : nullptr;
  aa.K = L.K;
  aa.bchunk = max(1, kAbsMaxRows / G);
  aa.sched = sched; aa.tile = L.tile; aa.G = L.G; aa.err = p.err;
  int nchunks = (B + aa.bchunk - 1) / aa.bchunk;
  size_t smem_abs = (size_t)aa.bchunk * G * p.dn * sizeof(float);
  absorb_kernel<T><<<cfg.n_kv_heads * nchunks + 1, 256, smem_abs, s>>>(aa);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 2. split-K attention over the latent cache
  if (L.kernel == 1) {
    DecodeArgs da;
    da.cache = c; da.B = B; da.H = H; da.n_kv = cfg.n_kv_heads; da.r = cfg.r_pairs;
    da.d_c = cfg.d_c; da.R = p.R; da.qlat = aa.qlat; da.qrope = aa.qrope;
    da.opart = (float*)(base + L.off_opart); da.mlpart = (float*)(base + L.off_mlpart);
    da.sched = sched;
    size_t smem = sizeof(float) * ((size_t)H * cfg.d_c + H * 2 * cfg.r_pairs +
                                   kSimtTile * (cfg.d_c + 1) + kSimtTile * (p.R + 1) +
                                   kSimtTile * H + 3 * H);
    e = cudaFuncSetAttribute(decode_simt_kernel<T, INT4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    if (p.opt_events) cudaEventRecord((cudaEvent_t)p.opt_events[0], s);
    decode_simt_kernel<T, INT4><<<L.G, 256, smem, s>>>(da);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.opt_events) cudaEventRecord((cudaEvent_t)p.opt_events[1], s);
  } else {
    if (p.opt_events) cudaEventRecord((cudaEvent_t)p.opt_events[0], s);
    e = mla_launch_decode_tc(p, c, B, sched, base + L.off_qlat, (float*)(base + L.off_opart),
                             (float*)(base + L.off_mlpart), L.G, s);
    if (e != cudaSuccess) return e;
    if (p.opt_events) cudaEventRecord((cudaEvent_t)p.opt_events[1], s);
  }
  // 3. merge the splits and apply W_uv
  CombineArgs ca;
  ca.B = B; ca.H = H; ca.n_kv = cfg.n_kv_heads; ca.d_c = cfg.d_c; ca.dh = cfg.head_dim;
  ca.opart = (const float*)(base + L.off_opart); ca.mlpart = (const float*)(base + L.off_mlpart);
  ca.sched = sched; ca.W_uv = p.W_uv; ca.out = out;
  ca.bchunk = max(1, 8 / G);
  int cchunks = (B + ca.bchunk - 1) / ca.bchunk;
  size_t smem_c = (size_t)ca.bchunk * G * (cfg.d_c + 2) * sizeof(float);
  combine_kernel<T><<<cfg.n_kv_heads * cchunks, 256, smem_c, s>>>(ca);
  return cudaGetLastError();
}

}  // namespace mla

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

DecodeLayout mla_decode_layout(const mla_plan& p, int B, int kernel) {
  const mla_config_t& cfg = p.cfg;
  DecodeLayout L;
  L.kernel = kernel;
  L.tile = kernel == 2 ? 64 : mla::kSimtTile;
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
  if (L.kernel == 1) {
    L.off_qlat = take(sizeof(float) * (size_t)B * H * cfg.d_c);
    L.off_qrope = take(sizeof(float) * (size_t)B * H * 2 * cfg.r_pairs + 4);
  } else {
    L.off_qlat = take(sizeof(uint16_t) * (size_t)B * H * L.K);
    L.off_qrope = L.off_qlat;
  }
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
