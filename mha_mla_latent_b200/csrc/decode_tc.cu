// Split-K latent attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Paper notes "MHA2MLA" (ACL 2025), §关键设计: all heads score against the one shared
// latent c_kv (W_uk absorbed into the query), the kept RoPE dims add a separate score
// term, and the value side is the probability-weighted latent taken through W_uv.
// Because every head reads the same c_kv row, the per-tile work is a real dense
// contraction: for a tile of 64 cached tokens
//     S[t][h]  = sum_k [C | KR][t][k] * Q'[h][k]          (MMA1, tokens on M, heads on N)
//     O[d][h] += sum_t C[t][d] * P[t][h]                  (MMA2, latent dims on M)
// where Q' is the absorbed query row [q_lat | block-diagonal q_rope] (bf16, pre-scaled
// by log2(e)/sqrt(d_h)), so the RoPE score is folded into MMA1 as K = d_c + n_kv*2r.
// MMA2 reuses the C tile already in shared memory as an MN-major A operand.
//
// One persistent CTA per SM walks its contiguous range of tiles (split-K schedule).
// Warp roles:
//   warp 0      TMA producer: Q' per piece; C and KR tiles into two rings of stages
//               (int4 cache: codes + scales into a raw ring instead of C)
//   warp 1      TMEM owner and single-thread MMA issuer; MMA1(n+1) is issued before
//               MMA2(n) so the tensor pipe works while the softmax of tile n finishes
//   warps 2-5   softmax: one TMEM lane (token) per thread, 32 heads per thread; online
//               softmax in log2 units with lazy rescaling (the running max is raised only
//               when a score exceeds it by more than 2^8, then O in TMEM is rescaled);
//               writes P (bf16) for MMA2; per-piece epilogue writes the partial (m, l, O)
//   warps 6-9   (int4 cache) dequantise codes*scale into the bf16 C stage
// Every wait is bounded (about 1 s); a timeout sets MLA_DEVERR_TIMEOUT, all roles stop,
// in-flight copies and MMAs are drained and TMEM is released before the CTA exits.
#include <cuda.h>

#include "decode_common.cuh"
#include "sm100.cuh"

namespace mla {
namespace tc {

using namespace sm100;

constexpr int kTile = 64;        // tokens per tile (MMA1 M)
constexpr int kH = 32;           // heads handled by this kernel (MMA N)
constexpr float kTau = 8.0f;     // lazy-rescale threshold, log2 units
constexpr uint32_t kBox = 8192;  // 64 rows x 128 B TMA box
constexpr uint32_t kQBox = 4096; // 32 rows x 128 B
constexpr uint32_t kPBytes = kTile * kH * 2;

struct TcArgs {
  int B, H, d_c, R, K, T_cap;
  Sched sched;
  float* opart;
  float* mlpart;
  const __half* scales;   // int4: [B*T_cap][d_c/32]
  int32_t* err;
  int NC, NK, NRAW;       // ring depths
  uint32_t off_c, off_kr, off_q, off_p, off_raw, off_bar, off_misc;  // from the 1024-aligned base
};

// barrier indices inside the barrier block
struct Bars {
  uint32_t base;
  int NC, NK, NRAW;
  __device__ uint32_t at(int i) const { return base + 8u * (uint32_t)i; }
  __device__ uint32_t c_full(int s) const { return at(s); }
  __device__ uint32_t c_empty(int s) const { return at(NC + s); }
  __device__ uint32_t kr_full(int s) const { return at(2 * NC + s); }
  __device__ uint32_t kr_empty(int s) const { return at(2 * NC + NK + s); }
  __device__ uint32_t raw_full(int s) const { return at(2 * NC + 2 * NK + s); }
  __device__ uint32_t raw_empty(int s) const { return at(2 * NC + 2 * NK + NRAW + s); }
  __device__ int fixed() const { return 2 * NC + 2 * NK + 2 * NRAW; }
  __device__ uint32_t q_full() const { return at(fixed() + 0); }
  __device__ uint32_t q_empty() const { return at(fixed() + 1); }
  __device__ uint32_t s_full(int i) const { return at(fixed() + 2 + i); }
  __device__ uint32_t s_empty(int i) const { return at(fixed() + 4 + i); }
  __device__ uint32_t p_full(int i) const { return at(fixed() + 6 + i); }
  __device__ uint32_t p_empty(int i) const { return at(fixed() + 8 + i); }
  __device__ uint32_t o_full(int i) const { return at(fixed() + 10 + i); }
  __device__ uint32_t o_empty(int i) const { return at(fixed() + 12 + i); }
  __device__ uint32_t grp(int i) const { return at(fixed() + 14 + i); }  // softmax-group syncs
  __device__ uint32_t mma_done() const { return at(fixed() + 16); }
  __device__ int count() const { return fixed() + 17; }
};

struct Misc {  // small shared scratch
  uint32_t tmem_base;
  int abort_flag;
  int vote[2][4];
  float red_max[2][4][kH];
  float red_sum[4][kH];
  float mt[4][kH];
};

// Per-worker iteration over (piece, tile) in schedule order.
struct TileIter {
  const Sched* s;
  int pc, pc_end;     // current piece, end
  int b, t0, t1;      // piece
  int t;              // current tile start (token)
  __device__ void init(const Sched* sc, int w) {
    s = sc;
    pc = sc->worker_first[w];
    pc_end = sc->worker_first[w + 1];
    t = 0;
    if (pc < pc_end) load();
  }
  __device__ void load() { b = s->piece_b[pc]; t0 = s->piece_t0[pc]; t1 = s->piece_t1[pc]; t = t0; }
  __device__ bool valid() const { return pc < pc_end; }
  __device__ bool first_of_piece() const { return t == t0; }
  __device__ bool last_of_piece() const { return t + kTile >= t1; }
  __device__ void next() {
    t += kTile;
    if (t >= t1) { ++pc; if (pc < pc_end) load(); }
  }
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ uint32_t f2u(float f) { return __float_as_uint(f); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// lane i ends with the reduction over the warp of element i (31 shuffles)
template <bool kMax>
__device__ __forceinline__ float transpose_reduce(float (&v)[kH], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int k = 0; k < off; ++k) {
      float send = upper ? v[k] : v[k + off];
      float keep = upper ? v[k + off] : v[k];
      float recv = __shfl_xor_sync(0xffffffffu, send, off);
      v[k] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return v[0];
}

template <bool INT4>
__global__ void __launch_bounds__(INT4 ? 320 : 192, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_kr,
                 const __grid_constant__ CUtensorMap tm_q, TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (sbase_u32 - smem_u32(smem_raw));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int dc = a.d_c, R = a.R, K = a.K;
  const int n_cbox = dc / 64, n_krbox = R / 64, n_qbox = K / 64;
  const uint32_t c_stage = (uint32_t)n_cbox * kBox, kr_stage = (uint32_t)n_krbox * kBox;
  const uint32_t raw_codes = (uint32_t)kTile * (dc / 2), raw_stage = raw_codes + (uint32_t)kTile * (dc / 16);
  const int nchunk = dc >= 128 ? dc / 128 : 1;      // MMA2 M-chunks (M = 128, or one M = 64)
  const int m2 = dc >= 128 ? 128 : 64;
  const uint32_t S_COL = 0, O_COL = 2 * kH, O_STRIDE = (uint32_t)nchunk * kH;
  Bars bars{sbase_u32 + a.off_bar, a.NC, a.NK, a.NRAW};
  Misc* misc = reinterpret_cast<Misc*>(sbase + a.off_misc);
  volatile int* abort_flag = &misc->abort_flag;

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    misc->abort_flag = 0;
    for (int s = 0; s < a.NC; ++s) {
      mbar_init(bars.c_full(s), INT4 ? 4 : 1);
      mbar_init(bars.c_empty(s), 1);
    }
    for (int s = 0; s < a.NK; ++s) { mbar_init(bars.kr_full(s), 1); mbar_init(bars.kr_empty(s), 1); }
    for (int s = 0; s < a.NRAW; ++s) { mbar_init(bars.raw_full(s), 1); mbar_init(bars.raw_empty(s), 4); }
    mbar_init(bars.q_full(), 1);
    mbar_init(bars.q_empty(), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars.s_full(i), 1);
      mbar_init(bars.s_empty(i), 4);
      mbar_init(bars.p_full(i), 4);
      mbar_init(bars.p_empty(i), 1);
      mbar_init(bars.o_full(i), 1);
      mbar_init(bars.o_empty(i), 4);
      mbar_init(bars.grp(i), 4);
    }
    mbar_init(bars.mma_done(), 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_kr);
    tma_prefetch_desc(&tm_q);
  }
  const uint32_t tmem_cols = (O_COL + 2 * O_STRIDE) <= 128 ? 128u : 256u;
  if (warp == 1) {
    tmem_alloc(smem_u32(&misc->tmem_base), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  const int w = blockIdx.x;

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      TileIter it;
      it.init(&a.sched, w);
      int n = 0, u = 0;
      int last_c = -1, last_kr = -1, last_raw = -1;
      int q_loads = 0;
      bool ok = true;
      while (ok && it.valid()) {
        if (it.first_of_piece()) {
          if (u > 0) ok = mbar_wait(bars.q_empty(), (u - 1) & 1, abort_flag);
          if (!ok) break;
          mbar_expect_tx(bars.q_full(), (uint32_t)n_qbox * kQBox);
          for (int kb = 0; kb < n_qbox; ++kb)
            tma_load_2d(sbase_u32 + a.off_q + kb * kQBox, &tm_q, bars.q_full(), kb * 64, it.b * a.H);
          ++q_loads;
        }
        const int row = it.b * a.T_cap + it.t;
        const int ks = n % a.NK;
        if (n >= a.NK) ok = mbar_wait(bars.kr_empty(ks), ((n / a.NK) - 1) & 1, abort_flag);
        if (!ok) break;
        mbar_expect_tx(bars.kr_full(ks), kr_stage);
        for (int rb = 0; rb < n_krbox; ++rb)
          tma_load_2d(sbase_u32 + a.off_kr + ks * kr_stage + rb * kBox, &tm_kr, bars.kr_full(ks), rb * 64, row);
        last_kr = n;
        if (!INT4) {
          const int cs = n % a.NC;
          if (n >= a.NC) ok = mbar_wait(bars.c_empty(cs), ((n / a.NC) - 1) & 1, abort_flag);
          if (!ok) break;
          mbar_expect_tx(bars.c_full(cs), c_stage);
          for (int cb = 0; cb < n_cbox; ++cb)
            tma_load_2d(sbase_u32 + a.off_c + cs * c_stage + cb * kBox, &tm_c, bars.c_full(cs), cb * 64, row);
          last_c = n;
        } else {
          const int rs = n % a.NRAW;
          if (n >= a.NRAW) ok = mbar_wait(bars.raw_empty(rs), ((n / a.NRAW) - 1) & 1, abort_flag);
          if (!ok) break;
          const int nvalid = min(kTile, it.t1 - it.t);
          const uint32_t sbytes = (uint32_t)((((nvalid + 1) & ~1) * (dc / 16) + 15) & ~15);
          mbar_expect_tx(bars.raw_full(rs), raw_codes + sbytes);
          tma_load_2d(sbase_u32 + a.off_raw + rs * raw_stage, &tm_c, bars.raw_full(rs), 0, row);
          bulk_load(sbase_u32 + a.off_raw + rs * raw_stage + raw_codes, a.scales + (size_t)row * (dc / 32), sbytes,
                    bars.raw_full(rs));
          last_raw = n;
        }
        if (it.last_of_piece()) ++u;
        it.next();
        ++n;
      }
      // drain: every issued copy must land before the CTA can exit
      volatile int never = 0;
      if (q_loads > 0) mbar_wait(bars.q_full(), (q_loads - 1) & 1, &never);
      for (int s = 0; s < a.NK; ++s) {
        int k = last_kr - ((last_kr - s) % a.NK + a.NK) % a.NK;  // last issue into slot s
        if (last_kr >= 0 && k >= 0) mbar_wait(bars.kr_full(s), (k / a.NK) & 1, &never);
      }
      if (!INT4) {
        for (int s = 0; s < a.NC; ++s) {
          int k = last_c - ((last_c - s) % a.NC + a.NC) % a.NC;
          if (last_c >= 0 && k >= 0) mbar_wait(bars.c_full(s), (k / a.NC) & 1, &never);
        }
      } else {
        for (int s = 0; s < a.NRAW; ++s) {
          int k = last_raw - ((last_raw - s) % a.NRAW + a.NRAW) % a.NRAW;
          if (last_raw >= 0 && k >= 0) mbar_wait(bars.raw_full(s), (k / a.NRAW) & 1, &never);
        }
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = idesc_bf16_f32(kTile, kH, false, false);
      const uint32_t idesc2 = idesc_bf16_f32(m2, kH, true, true);
      TileIter it;
      it.init(&a.sched, w);
      int n = 0, u = 0;
      bool ok = true;
      // state of the tile whose MMA2 is pending
      int pend_n = -1, pend_u = 0;
      bool pend_first = false, pend_last = false;
      auto do_mma2 = [&](int pn, int pu, bool first, bool last) -> bool {
        const int pb = pn & 1, cs = pn % a.NC, ob = pu & 1;
        if (!mbar_wait(bars.p_full(pb), (pn >> 1) & 1, abort_flag)) return false;
        if (first && pu >= 2)
          if (!mbar_wait(bars.o_empty(ob), ((pu >> 1) - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t c0 = sbase_u32 + a.off_c + cs * c_stage;
        const uint32_t p0 = sbase_u32 + a.off_p + pb * kPBytes;
        for (int mc = 0; mc < nchunk; ++mc) {
          const uint32_t d = tmem + O_COL + ob * O_STRIDE + mc * kH;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            uint64_t ad = smem_desc(c0 + mc * 2 * kBox + kk * 2048, kBox, 1024, kLayoutSW128);
            uint64_t bd = smem_desc(p0 + kk * 256, 128, 1024, kLayoutNone);
            tc_mma_bf16(d, ad, bd, idesc2, (first && kk == 0) ? 0u : 1u);
          }
        }
        tc_commit(bars.p_empty(pb));
        tc_commit(bars.c_empty(cs));
        if (last) tc_commit(bars.o_full(ob));
        return true;
      };
      while (ok && it.valid()) {
        const int sb = n & 1, cs = n % a.NC, ks = n % a.NK;
        if (n >= 2) ok = mbar_wait(bars.s_empty(sb), ((n >> 1) - 1) & 1, abort_flag);
        if (ok && it.first_of_piece()) ok = mbar_wait(bars.q_full(), u & 1, abort_flag);
        if (ok) ok = mbar_wait(bars.kr_full(ks), (n / a.NK) & 1, abort_flag);
        if (ok) ok = mbar_wait(bars.c_full(cs), (n / a.NC) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        {  // MMA1: S = [C | KR] Q'^T
          const uint32_t d = tmem + S_COL + sb * kH;
          const uint32_t c0 = sbase_u32 + a.off_c + cs * c_stage;
          const uint32_t k0 = sbase_u32 + a.off_kr + ks * kr_stage;
          const uint32_t q0 = sbase_u32 + a.off_q;
          for (int kk = 0; kk < dc / 16; ++kk) {
            uint64_t ad = smem_desc(c0 + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024, kLayoutSW128);
            uint64_t bd = smem_desc(q0 + (kk >> 2) * kQBox + (kk & 3) * 32, 16, 1024, kLayoutSW128);
            tc_mma_bf16(d, ad, bd, idesc1, kk > 0 ? 1u : 0u);
          }
          for (int kk = 0; kk < R / 16; ++kk) {
            uint64_t ad = smem_desc(k0 + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024, kLayoutSW128);
            uint64_t bd = smem_desc(q0 + (n_cbox + (kk >> 2)) * kQBox + (kk & 3) * 32, 16, 1024, kLayoutSW128);
            tc_mma_bf16(d, ad, bd, idesc1, 1u);
          }
          tc_commit(bars.s_full(sb));
          tc_commit(bars.kr_empty(ks));
          if (it.last_of_piece()) tc_commit(bars.q_empty());
        }
        if (pend_n >= 0) {
          ok = do_mma2(pend_n, pend_u, pend_first, pend_last);
          if (!ok) break;
        }
        pend_n = n; pend_u = u; pend_first = it.first_of_piece(); pend_last = it.last_of_piece();
        if (it.last_of_piece()) ++u;
        it.next();
        ++n;
      }
      if (ok && pend_n >= 0) do_mma2(pend_n, pend_u, pend_first, pend_last);
      // drain: all issued MMAs complete before TMEM is released
      tc_commit(bars.mma_done());
      volatile int never = 0;
      mbar_wait(bars.mma_done(), 0, &never);
    }
  } else if (warp < 6) {
    // ============================================================ softmax + epilogue
    const int q = warp & 3;            // TMEM lane quarter of this warp
    const int row = 16 * q + lane;     // token row within the tile (M = 64 layout), lane < 16
    TileIter it;
    it.init(&a.sched, w);
    int n = 0, u = 0, gphase0 = 0, gphase1 = 0;
    bool ok = true;
    float m[kH], l[kH];
    auto wwait = [&](uint32_t bar, int parity) -> bool {  // warp-uniform outcome
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    auto grp_sync = [&](int i) -> bool {  // all 4 softmax warps, bounded
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.grp(i));
      int& ph = i ? gphase1 : gphase0;
      bool r = wwait(bars.grp(i), ph & 1);
      ++ph;
      return r;
    };
    while (ok && it.valid()) {
      const int pc = it.pc;
      const bool first = it.first_of_piece();
      if (first) {
#pragma unroll
        for (int h = 0; h < kH; ++h) { m[h] = -INFINITY; l[h] = 0.f; }
      }
      const int sb = n & 1, pb = n & 1, ob = u & 1;
      const int nvalid = min(kTile, it.t1 - it.t);
      const bool valid = lane < 16 && row < nvalid;
      ok = wwait(bars.s_full(sb), (n >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      float v[kH];
      {
        uint32_t raw[32];
        tmem_ld32(taddr(tmem, 32 * q, S_COL + sb * kH), raw);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < kH; ++h) v[h] = valid ? u2f(raw[h]) : -INFINITY;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.s_empty(sb));
      // does any score exceed its head's running max by more than tau?
      bool need = false;
      if (valid) {
#pragma unroll
        for (int h = 0; h < kH; ++h) need |= (v[h] - m[h] > kTau);
      }
      need = __any_sync(0xffffffffu, need);
      if (lane == 0) misc->vote[n & 1][q] = need ? 1 : 0;
      ok = grp_sync(0);
      if (!ok) break;
      const bool need_all = misc->vote[n & 1][0] | misc->vote[n & 1][1] | misc->vote[n & 1][2] | misc->vote[n & 1][3];
      if (need_all) {
        float t[kH];
#pragma unroll
        for (int h = 0; h < kH; ++h) t[h] = v[h];
        const float wmax = transpose_reduce<true>(t, lane);
        misc->red_max[n & 1][q][lane] = wmax;
        ok = grp_sync(1);
        if (!ok) break;
        float mt = fmaxf(fmaxf(misc->red_max[n & 1][0][lane], misc->red_max[n & 1][1][lane]),
                         fmaxf(misc->red_max[n & 1][2][lane], misc->red_max[n & 1][3][lane]));
        misc->mt[q][lane] = mt;
        __syncwarp();
        float alpha[kH];
        bool any_scale = false;
#pragma unroll
        for (int h = 0; h < kH; ++h) {
          const float mn = fmaxf(m[h], misc->mt[q][h]);
          alpha[h] = exp2f(m[h] - mn);   // m = -inf on a piece's first tile -> 0
          any_scale |= (mn != m[h]);
          m[h] = mn;
          l[h] *= alpha[h];
        }
        if (!first && any_scale) {
          // O holds tiles < n of this piece: wait for MMA2(n-1), rescale the columns
          const int pn = n - 1;
          ok = wwait(bars.p_empty(pn & 1), (pn >> 1) & 1);
          if (!ok) break;
          tc_fence_after();
          for (int mc = 0; mc < nchunk; ++mc) {
            const uint32_t ta = taddr(tmem, 32 * q, O_COL + ob * O_STRIDE + mc * kH);
            uint32_t o[32];
            tmem_ld32(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < kH; ++h) o[h] = f2u(u2f(o[h]) * alpha[h]);
            tmem_st32(ta, o);
          }
          tmem_wait_st();
        }
      }
      // probabilities for this tile
      uint32_t pk[kH / 2];
#pragma unroll
      for (int h = 0; h < kH; h += 2) {
        const float p0 = valid ? exp2f(v[h] - m[h]) : 0.f;
        const float p1 = valid ? exp2f(v[h + 1] - m[h + 1]) : 0.f;
        l[h] += p0;
        l[h + 1] += p1;
        pk[h / 2] = pack_bf16x2(p0, p1);
      }
      if (n >= 2) {
        ok = wwait(bars.p_empty(pb), ((n - 2) >> 1) & 1);
        if (!ok) break;
      }
      if (lane < 16) {
        // P as the MN-major (heads contiguous) B operand, no swizzle: core matrices of
        // 8 heads x 8 tokens; head block at 1024 B, token block at 128 B.
        uint8_t* P = sbase + a.off_p + pb * kPBytes + (row >> 3) * 128 + (row & 7) * 16;
#pragma unroll
        for (int hb = 0; hb < 4; ++hb)
          *reinterpret_cast<uint4*>(P + hb * 1024) =
              make_uint4(pk[4 * hb], pk[4 * hb + 1], pk[4 * hb + 2], pk[4 * hb + 3]);
        if (!INT4 && row >= nvalid) {
          // rows past the sequence end: clear the latent row so MMA2 never multiplies
          // stale cache contents (0 * NaN would poison O)
          uint8_t* C = sbase + a.off_c + (n % a.NC) * c_stage + row * 128;
          for (int cb = 0; cb < n_cbox; ++cb)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(C + cb * kBox + ch * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full(pb));

      if (it.last_of_piece()) {
        // ---------------- piece epilogue: partial (m, l, O) for the split merge
        float t[kH];
#pragma unroll
        for (int h = 0; h < kH; ++h) t[h] = (lane < 16) ? l[h] : 0.f;
        const float lsum = transpose_reduce<false>(t, lane);
        misc->red_sum[q][lane] = lsum;
        ok = grp_sync(1);
        if (!ok) break;
        if (q == 0) {
          const float L = misc->red_sum[0][lane] + misc->red_sum[1][lane] + misc->red_sum[2][lane] +
                          misc->red_sum[3][lane];
          float mh = m[0];
#pragma unroll
          for (int h = 1; h < kH; ++h) mh = (lane == h) ? m[h] : mh;
          a.mlpart[((size_t)pc * kH + lane) * 2] = mh;
          a.mlpart[((size_t)pc * kH + lane) * 2 + 1] = L;
        }
        ok = wwait(bars.o_full(ob), (u >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        for (int mc = 0; mc < nchunk; ++mc) {
          uint32_t o[32];
          tmem_ld32(taddr(tmem, 32 * q, O_COL + ob * O_STRIDE + mc * kH), o);
          tmem_wait_ld();
          int d;
          bool dv;
          if (m2 == 128) { d = mc * 128 + 32 * q + lane; dv = true; }
          else { d = 16 * q + lane; dv = lane < 16; }
          if (dv) {
            float* dst = a.opart + (size_t)pc * kH * dc + d;
#pragma unroll
            for (int h = 0; h < kH; ++h) dst[(size_t)h * dc] = u2f(o[h]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.o_empty(ob));
        ++u;
      }
      it.next();
      ++n;
    }
  } else if (INT4) {
    // ============================================================ int4 dequantisation
    const int dw = warp - 6;
    const int tok = dw * 16 + (lane & 15);
    const int half = lane >> 4;                 // which 64-wide box of the 128-wide latent
    TileIter it;
    it.init(&a.sched, w);
    int n = 0;
    bool ok = true;
    while (ok && it.valid()) {
      const int rs = n % a.NRAW, cs = n % a.NC;
      ok = __all_sync(0xffffffffu, mbar_wait(bars.raw_full(rs), (n / a.NRAW) & 1, abort_flag));
      if (ok && n >= a.NC)
        ok = __all_sync(0xffffffffu, mbar_wait(bars.c_empty(cs), ((n / a.NC) - 1) & 1, abort_flag));
      if (!ok) break;
      const int nvalid = min(kTile, it.t1 - it.t);
      const uint8_t* raw = sbase + a.off_raw + rs * raw_stage;
      uint8_t* C = sbase + a.off_c + cs * c_stage + half * kBox + tok * 128;
      if (tok < nvalid) {
        const uint4 c0 = *reinterpret_cast<const uint4*>(raw + tok * (dc / 2) + half * 32);
        const uint4 c1 = *reinterpret_cast<const uint4*>(raw + tok * (dc / 2) + half * 32 + 16);
        const __half* sc = reinterpret_cast<const __half*>(raw + raw_codes) + tok * (dc / 32) + half * 2;
        const float s0 = __half2float(sc[0]), s1 = __half2float(sc[1]);
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {           // 8 latent values per 16-byte chunk
          const uint32_t wd = words[ch];
          const float s = ch < 4 ? s0 : s1;
          uint32_t o[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t byte = (wd >> (8 * j)) & 0xFFu;
            o[j] = pack_bf16x2((float)nib_to_int(byte & 15u) * s, (float)nib_to_int(byte >> 4) * s);
          }
          *reinterpret_cast<uint4*>(C + ((ch ^ (tok & 7)) * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      } else {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(C + ch * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bars.raw_empty(rs));
        mbar_arrive(bars.c_full(cs));
      }
      it.next();
      ++n;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
  if (threadIdx.x == 0 && misc->abort_flag) raise_error(a.err, MLA_DEVERR_TIMEOUT);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

static bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t cols, uint64_t rows,
                        uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {row_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), gdim, gstride, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct TcLayout {
  int NC, NK, NRAW;
  uint32_t off_c, off_kr, off_q, off_p, off_raw, off_bar, off_misc, total;
};

static TcLayout tc_layout(int dc, int R, int K, bool int4) {
  const uint32_t budget = 232448 - 1024;  // max dynamic smem per block minus alignment slack
  const uint32_t c_stage = (uint32_t)(dc / 64) * kBox, kr_stage = (uint32_t)(R / 64) * kBox;
  const uint32_t raw_stage = (uint32_t)kTile * (dc / 2) + (uint32_t)kTile * (dc / 16);
  const uint32_t q_bytes = (uint32_t)(K / 64) * kQBox;
  TcLayout L{};
  auto size = [&](int nc, int nk, int nraw) {
    uint32_t s = nc * c_stage + nk * kr_stage + q_bytes + 2 * kPBytes;
    s += int4 ? ((nraw * raw_stage + 1023) & ~1023u) : 0;
    s += 8 * (2 * nc + 2 * nk + 2 * nraw + 17) + sizeof(Misc) + 64;
    return s;
  };
  int nc = 2, nk = 2, nraw = int4 ? 2 : 0;
  for (int it = 0; it < 12; ++it) {  // grow the rings while they fit, KR first (largest stream)
    bool grew = false;
    if (nk < 6 && size(nc, nk + 1, nraw) <= budget) { ++nk; grew = true; }
    if (int4 && nraw < 6 && size(nc, nk, nraw + 1) <= budget) { ++nraw; grew = true; }
    if (nc < 6 && size(nc + 1, nk, nraw) <= budget) { ++nc; grew = true; }
    if (!grew) break;
  }
  L.NC = nc; L.NK = nk; L.NRAW = nraw;
  uint32_t o = 0;
  L.off_c = o; o += nc * c_stage;
  L.off_kr = o; o += nk * kr_stage;
  L.off_q = o; o += q_bytes;
  L.off_p = o; o += 2 * kPBytes;
  L.off_raw = o; o += int4 ? ((nraw * raw_stage + 1023) & ~1023u) : 0;
  L.off_bar = o; o += 8 * (2 * nc + 2 * nk + 2 * nraw + 17);
  o = (o + 15) & ~15u;
  L.off_misc = o; o += sizeof(Misc);
  L.total = o + 1024;
  return L;
}

}  // namespace tc
}  // namespace mla

// Shapes the tensor-core kernel covers: bf16, 32 heads, d_c in {64, 128, 256}, RoPE
// width a multiple of 64; the int4 cache with d_c = 128.
bool mla_tc_capable(const mla_plan& p) {
  const mla_config_t& cfg = p.cfg;
  if (cfg.dtype != MLA_BF16 || cfg.n_heads != mla::tc::kH) return false;
  if (cfg.d_c % 64 != 0 || cfg.d_c > 256 || p.R % 64 != 0 || p.R == 0) return false;
  if (cfg.cache_kind == MLA_CACHE_INT4_G32 && cfg.d_c != 128) return false;
  return true;
}

// The int4 scale rows are fetched with 1-D bulk copies, which need an even capacity.
bool mla_tc_supported(const mla_plan& p, const mla_cache_t& c) {
  if (!mla_tc_capable(p)) return false;
  if (p.cfg.cache_kind == MLA_CACHE_INT4_G32 && c.T_cap % 2 != 0) return false;
  return true;
}

cudaError_t mla_launch_decode_tc(const mla_plan& p, const mla_cache_t& c, int B, const Sched& sched,
                                 const void* qcat, float* opart, float* mlpart, int G, cudaStream_t s) {
  using namespace mla::tc;
  const mla_config_t& cfg = p.cfg;
  const bool int4 = cfg.cache_kind == MLA_CACHE_INT4_G32;
  const int dc = cfg.d_c, R = p.R, K = dc + R;
  CUtensorMap tm_c, tm_kr, tm_q;
  const uint64_t rows = (uint64_t)c.B * c.T_cap;
  bool ok = true;
  if (int4)
    ok &= make_map_2d(&tm_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.c_kv, dc / 2, rows, dc / 2, dc / 2, kTile,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    ok &= make_map_2d(&tm_c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c.c_kv, dc, rows, (uint64_t)dc * 2, 64, kTile,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_2d(&tm_kr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c.k_rope, R, rows, (uint64_t)R * 2, 64, kTile,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qcat, K, (uint64_t)B * kH, (uint64_t)K * 2, 64, kH,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  TcLayout L = tc_layout(dc, R, K, int4);
  TcArgs a;
  a.B = B; a.H = kH; a.d_c = dc; a.R = R; a.K = K; a.T_cap = c.T_cap;
  a.sched = sched; a.opart = opart; a.mlpart = mlpart;
  a.scales = (const __half*)c.c_scales; a.err = p.err;
  a.NC = L.NC; a.NK = L.NK; a.NRAW = L.NRAW;
  a.off_c = L.off_c; a.off_kr = L.off_kr; a.off_q = L.off_q; a.off_p = L.off_p; a.off_raw = L.off_raw;
  a.off_bar = L.off_bar; a.off_misc = L.off_misc;
  auto kern = int4 ? decode_tc_kernel<true> : decode_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  kern<<<G, int4 ? 320 : 192, L.total, s>>>(tm_c, tm_kr, tm_q, a);
  return cudaGetLastError();
}
