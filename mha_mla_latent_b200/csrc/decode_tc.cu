// Split-K latent attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Paper notes "MHA2MLA" (ACL 2025), §关键设计: all heads score against the one shared
// latent c_kv (W_uk absorbed into the query), the kept RoPE dims add a separate score
// term that cannot join the matrix merge, and the value side is the probability-weighted
// latent taken through W_uv.  Because every head reads the same c_kv row, the per-tile
// work is a real dense contraction.  For a tile of 128 cached tokens of one sequence:
//     S[t][h]   = sum_c C[t][c] * Qlat[h][c]            MMA1  M = 128 tokens, N = 32 heads
//     S[t][h]  += sum_j KR[t][g(h)][j] * Qrope[h][j]    CUDA cores (fp32)
//     O^T[h][d] += sum_t P^T[h][t] * C[t][d]            MMA2  M = 64 (32 heads + pad), N = d_c
// MMA2 reuses the C tile already in shared memory as an MN-major B operand, so each
// cached byte is read from HBM once.  The RoPE term has 8 dims per head; as extra K of
// MMA1 it would double the MMAs per tile, so it runs on the CUDA cores beside them.
//
// One persistent CTA per SM walks its contiguous range of tiles (split-K schedule).
// Warp roles (12 warps, three warpgroups; setmaxnreg gives warpgroups 1-2 224 registers):
//   warp 0      TMA producer: Q_lat per piece, C tiles into a ring of stages (int4 cache:
//               codes + scales into a raw ring instead)
//   warp 1      TMEM owner and single-thread MMA issuer; it polls and issues MMA2 of the
//               pending tile as soon as its P^T is ready, else MMA1 of the next tile
//   warps 2-3   (int4 cache) dequantise codes*scale into the bf16 C stage
//   warps 4-11  softmax: one token per thread (TMEM lane), 16 heads per thread (two warps
//               per lane quarter); RoPE keys from a bulk-copied stage via registers, the
//               RoPE score, online softmax in log2 units with lazy rescaling (the running
//               max is raised only when a score exceeds it by more than 2^8, then the O
//               rows are rescaled in TMEM), P^T (bf16) for MMA2, and per piece the
//               partial (m, l, O) for the split merge
// Every wait is bounded (about 1 s); a timeout sets MLA_DEVERR_TIMEOUT, all roles stop,
// in-flight copies and MMAs are drained and TMEM is released before the CTA exits.
#include <cuda.h>

#include "decode_common.cuh"
#include "sm100.cuh"

namespace mla {
namespace tc {

using namespace sm100;

constexpr int kTile = 128;          // tokens per tile
constexpr int kH = 32;              // heads handled by this kernel
constexpr int kHh = 16;             // heads per softmax warp (two warps per TMEM lane quarter)
constexpr int kSoftWarps = 8;
constexpr float kTau = 8.0f;        // lazy-rescale threshold, log2 units
constexpr uint32_t kBox = 16384;    // TMA box: 128 rows x 128 B (C, KR)
constexpr uint32_t kQBox = 4096;    // Q_lat box: 32 rows x 128 B
constexpr uint32_t kPtAtom = 8192;  // P^T: 64 rows x 128 B per 64-token atom
constexpr uint32_t kPtBytes = 2 * kPtAtom;

struct TcArgs {
  int B, H, d_c, R, r2, T_cap, P;
  Sched sched;
  float* opart;           // [P][H][d_c]
  float* mlpart;          // [H][P][2]
  const float* qrope;     // [B][H][2r] rotated, scaled RoPE query part
  const __half* scales;   // int4: [B*T_cap][d_c/32]
  const int32_t* seq_lens;            // residual window only
  mla_cache_t cache;                  // block table (paged cache) and geometry
  const __nv_bfloat16* c_resid;       // int4 with the residual window: [B][128][d_c], else null
  const int32_t* resid_pos;           // [B][128]
  const uint8_t* kr_base;
  uint32_t c_row, kr_row;
  int32_t* err;
  uint64_t wait_ns;       // bound of every pipeline wait
  int skip_tile;          // testing only: 1-based tile whose latent copy is left out (0 = none)
  int NC, NRAW, NP, NO;  // ring depths; P^T and O buffers
  uint32_t off_c, off_q, off_p, off_raw, off_qr, off_bar, off_misc;
  uint32_t off_kr;        // RoPE key stage: one tile, 4 blocks of [n_kv][32][2r]
};

struct Bars {
  uint32_t base;
  int NC, NRAW, NP, NO;
  __device__ uint32_t at(int i) const { return base + 8u * (uint32_t)i; }
  __device__ uint32_t c_full(int s) const { return at(s); }
  __device__ uint32_t c_empty(int s) const { return at(NC + s); }
  __device__ uint32_t raw_full(int s) const { return at(2 * NC + s); }
  __device__ uint32_t raw_empty(int s) const { return at(2 * NC + NRAW + s); }
  __device__ int o1() const { return 2 * NC + 2 * NRAW; }
  __device__ uint32_t p_full(int i) const { return at(o1() + i); }
  __device__ uint32_t p_empty(int i) const { return at(o1() + 2 + i); }
  __device__ uint32_t o_full(int i) const { return at(o1() + 4 + i); }
  __device__ uint32_t o_empty(int i) const { return at(o1() + 6 + i); }
  __device__ uint32_t s_full(int i) const { return at(o1() + 8 + i); }
  __device__ uint32_t s_empty(int i) const { return at(o1() + 10 + i); }
  __device__ uint32_t q_full() const { return at(o1() + 12); }
  __device__ uint32_t q_empty() const { return at(o1() + 13); }
  __device__ uint32_t grp(int i) const { return at(o1() + 14 + i); }
  __device__ uint32_t mma_done() const { return at(o1() + 16); }
  __device__ uint32_t kr_full() const { return at(o1() + 17); }
};
constexpr int kFixedBars = 18;

struct Misc {  // small shared scratch
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float red_max[2][4][kH];   // per tile parity, quarter, head: the warp's max score
  alignas(16) float red_l[4][kH];          // (read as float4)
  int kr_released;   // softmax warps done with the RoPE key stage (the 8th issues the next copy)
  int kr_issued;     // RoPE key copies issued
};

// Per-worker iteration over (piece, tile) in schedule order.
struct TileIter {
  const Sched* s;
  int pc, pc_end;
  int b, t0, t1;
  int t;
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
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Maximum over the warp (sm_100 warp-wide float reduction).
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Reduction over the 32 lanes of each of 16 values (15 + 1 shuffles): lanes i and i ^ 16
// end with the result for element (i & 15).
template <bool kMax>
__device__ __forceinline__ float transpose_reduce16(float (&v)[16], int lane) {
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int k = 0; k < off; ++k) {
      float send = upper ? v[k] : v[k + off];
      float keep = upper ? v[k + off] : v[k];
      float recv = __shfl_xor_sync(0xffffffffu, send, off);
      v[k] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  const float other = __shfl_xor_sync(0xffffffffu, v[0], 16);
  return kMax ? fmaxf(v[0], other) : v[0] + other;
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


// Storage location of (b, t): compile-time contiguous, or through the paged block table.
template <bool PAGED>
__device__ __forceinline__ MlaLoc tc_loc(const TcArgs& a, int b, int t) {
  if (!PAGED) return MlaLoc{b, t, a.T_cap};
  return mla_loc(a.cache, b, t, a.err);
}

// QB: code width of a quantised latent cache (4 or 2; dequantised in shared memory), 0 for a
// bf16 latent; RESID: with the residual window ring (4-bit only); PAGED: cache addressed
// through a block table.  Each combination is its own instantiation, so the common ones
// carry no code of the others.
template <int QB, bool RESID, bool PAGED, int R2>
__global__ void __launch_bounds__(384, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (sbase_u32 - smem_u32(smem_raw));
  constexpr bool INT4 = QB != 0;   // quantised latent (4- or 2-bit codes)
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int dc = a.d_c, R = a.R;
  const int n_cbox = dc / 64;
  const uint32_t c_stage = (uint32_t)n_cbox * kBox;
  constexpr int kCodeBytes64 = QB * 8;   // code bytes of 64 latent values
  const uint32_t raw_codes = (uint32_t)kTile * (dc / 64) * kCodeBytes64, raw_stage = raw_codes + (uint32_t)kTile * (dc / 16);
  const uint32_t S_COL = 0, O_COL = 2 * kH;
  Bars bars{sbase_u32 + a.off_bar, a.NC, a.NRAW, a.NP, a.NO};
  Misc* misc = reinterpret_cast<Misc*>(sbase + a.off_misc);
  volatile int* abort_flag = &misc->abort_flag;
  float* qr_s = reinterpret_cast<float*>(sbase + a.off_qr);   // [32][2r]
  // Q_lat boxes 0 and 1 live in the padding rows (32..63) of P^T buffer 0: MMA2 reads those
  // rows only into output rows that are never used; further boxes follow at off_q
  auto qbox = [&](int kb) -> uint32_t {
    return sbase_u32 + (kb < 2 ? a.off_p + 4096u + kPtAtom * kb : a.off_q + kQBox * (kb - 2));
  };

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    misc->abort_flag = 0;
    for (int s = 0; s < a.NC; ++s) { mbar_init(bars.c_full(s), INT4 ? 2 : 1); mbar_init(bars.c_empty(s), 1); }
    for (int s = 0; s < a.NRAW; ++s) { mbar_init(bars.raw_full(s), 1); mbar_init(bars.raw_empty(s), 2); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars.p_full(i), kSoftWarps);
      mbar_init(bars.p_empty(i), 1);
      mbar_init(bars.o_full(i), 1);
      mbar_init(bars.o_empty(i), kSoftWarps);
      mbar_init(bars.s_full(i), 1);
      mbar_init(bars.s_empty(i), kSoftWarps);
      mbar_init(bars.grp(i), kSoftWarps);
    }
    mbar_init(bars.q_full(), 1);
    mbar_init(bars.q_empty(), 1);
    mbar_init(bars.mma_done(), 1);
    mbar_init(bars.kr_full(), 1);
    misc->kr_released = 0;
    misc->kr_issued = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kr);
  }
  const uint32_t tmem_cols = (O_COL + a.NO * dc) <= 256 ? 256u : 512u;
  if (warp == 1) {
    tmem_alloc(smem_u32(&misc->tmem_base), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the schedule, absorbed queries and the cache come from earlier kernels
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem = misc->tmem_base;
  const int w = blockIdx.x;
  const uint64_t lim = a.wait_ns;

  // register split: the control warpgroup (producer, MMA issuer, int4 dequant) gives up
  // registers to the two softmax warpgroups: 128 * 56 + 256 * 224 = 384 * 168 at launch
  if (warp < 4) {
    setmaxnreg_dec<56>();
    if (warp == 0) {
      // ============================================================ TMA producer
      if (lane == 0) {
        TileIter it;
        it.init(&a.sched, w);
        int n = 0, u = 0, q_loads = 0;
        int last = -1, skipped = -1;
        bool ok = true;
        while (ok && it.valid()) {
          if (it.first_of_piece()) {
            if (u > 0) ok = mbar_wait(bars.q_empty(), (u - 1) & 1, abort_flag, lim);
            if (!ok) break;
            mbar_expect_tx(bars.q_full(), (uint32_t)n_cbox * kQBox);
            for (int kb = 0; kb < n_cbox; ++kb)
              tma_load_2d(qbox(kb), &tm_q, bars.q_full(), kb * 64, it.b * a.H);
            ++q_loads;
          }
          const MlaLoc lc = tc_loc<PAGED>(a, it.b, it.t);   // a tile is one paged block
          const int row = lc.pb * lc.cap + lc.pt;
          // testing hook (off unless set): leave this tile's latent copy out, so the waits
          // on it run out and the kernel reports MLA_DEVERR_TIMEOUT
          const bool skip = (n + 1 == a.skip_tile);
          if (!INT4) {
            const int cs = n % a.NC;
            if (n >= a.NC) ok = mbar_wait(bars.c_empty(cs), ((n / a.NC) - 1) & 1, abort_flag, lim);
            if (!ok) break;
            if (!skip) {
              mbar_expect_tx(bars.c_full(cs), c_stage);
              for (int cb = 0; cb < n_cbox; ++cb)
                tma_load_2d(sbase_u32 + a.off_c + cs * c_stage + cb * kBox, &tm_c, bars.c_full(cs), cb * 64, row);
            }
          } else {
            const int rs = n % a.NRAW;
            if (n >= a.NRAW) ok = mbar_wait(bars.raw_empty(rs), ((n / a.NRAW) - 1) & 1, abort_flag, lim);
            if (!ok) break;
            const int nvalid = min(kTile, it.t1 - it.t);
            const uint32_t sbytes = (uint32_t)((((nvalid + 1) & ~1) * (dc / 16) + 15) & ~15);
            if (!skip) {
              mbar_expect_tx(bars.raw_full(rs), raw_codes + sbytes);
              tma_load_2d(sbase_u32 + a.off_raw + rs * raw_stage, &tm_c, bars.raw_full(rs), 0, row);
              bulk_load(sbase_u32 + a.off_raw + rs * raw_stage + raw_codes, a.scales + (size_t)row * (dc / 32),
                        sbytes, bars.raw_full(rs));
            }
          }
          last = n;
          if (skip) skipped = n;
          if (it.last_of_piece()) ++u;
          it.next();
          ++n;
        }
        // drain: every issued copy must land before the CTA can exit (a skipped copy's
        // stage waits for the copy before it instead)
        volatile int never = 0;
        if (q_loads > 0) mbar_wait(bars.q_full(), (q_loads - 1) & 1, &never, lim);
        const int NS = INT4 ? a.NRAW : a.NC;
        for (int s = 0; s < NS; ++s) {
          int k = last - ((last - s) % NS + NS) % NS;
          if (k == skipped) k -= NS;
          if (last >= 0 && k >= 0) mbar_wait(INT4 ? bars.raw_full(s) : bars.c_full(s), (k / NS) & 1, &never, lim);
        }
      }
    } else if (warp == 1) {
      // ============================================================ MMA issuer
      if (lane == 0) {
        const uint32_t idesc1 = idesc_bf16_f32(kTile, kH, false, false);  // S[t][h]
        const uint32_t idesc2 = idesc_bf16_f32(64, dc, false, true);      // O^T[h][d]
        TileIter it;
        it.init(&a.sched, w);
        int n = 0, u = 0;
        bool ok = true;
        int pend_n = -1, pend_u = 0;
        bool pend_first = false, pend_last = false;
        auto do_mma2 = [&](int pn, int pu, bool first, bool last) -> bool {
          const int pb = pn % a.NP, cs = pn % a.NC, ob = pu % a.NO;
          if (!mbar_wait(bars.p_full(pb), (pn / a.NP) & 1, abort_flag, lim)) return false;
          if (first && pu >= a.NO)
            if (!mbar_wait(bars.o_empty(ob), ((pu / a.NO) - 1) & 1, abort_flag, lim)) return false;
          tc_fence_after();
          const uint32_t c0 = sbase_u32 + a.off_c + cs * c_stage;
          const uint32_t p0 = sbase_u32 + a.off_p + pb * kPtBytes;
          const uint32_t d = tmem + O_COL + ob * dc;
  #pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint64_t ad = smem_desc(p0 + (kk >> 2) * kPtAtom + (kk & 3) * 32, 16, 1024, kLayoutSW128);
            const uint64_t bd = smem_desc(c0 + kk * 2048, kBox, 1024, kLayoutSW128);
            tc_mma_bf16(d, ad, bd, idesc2, (first && kk == 0) ? 0u : 1u);
          }
          tc_commit(bars.p_empty(pb));
          tc_commit(bars.c_empty(cs));
          if (last) tc_commit(bars.o_full(ob));
          return true;
        };
        while (ok && it.valid()) {
          const int sb = n & 1, cs = n % a.NC;
          const bool first = it.first_of_piece();
          // MMA1(n) needs its S buffer free, the piece's Q_lat and the latent tile; MMA2 of the
          // pending tile needs its P^T.  Whichever is ready first goes first, so a pending tile
          // releases its latent stage (and the next copy can start) as early as possible.
          {
            const uint64_t t_start = globaltimer();
            while (true) {
              if (pend_n >= 0 && mbar_test(bars.p_full(pend_n % a.NP), (pend_n / a.NP) & 1)) {
                ok = do_mma2(pend_n, pend_u, pend_first, pend_last);
                pend_n = -1;
                if (!ok) break;
                continue;
              }
              if ((n < 2 || mbar_test(bars.s_empty(sb), ((n >> 1) - 1) & 1)) &&
                  (!first || mbar_test(bars.q_full(), u & 1)) && mbar_test(bars.c_full(cs), (n / a.NC) & 1))
                break;
              if (*abort_flag || globaltimer() - t_start > lim) {
                *abort_flag = 1;
                ok = false;
                break;
              }
            }
          }
          if (!ok) break;
          tc_fence_after();
          {  // MMA1: S = C Q_lat^T
            const uint32_t d = tmem + S_COL + sb * kH;
            const uint32_t c0 = sbase_u32 + a.off_c + cs * c_stage;
            for (int kk = 0; kk < dc / 16; ++kk) {
              const uint64_t ad = smem_desc(c0 + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024, kLayoutSW128);
              const uint64_t bd = smem_desc(qbox(kk >> 2) + (kk & 3) * 32, 16, 1024, kLayoutSW128);
              tc_mma_bf16(d, ad, bd, idesc1, kk > 0 ? 1u : 0u);
            }
            tc_commit(bars.s_full(sb));
            if (it.last_of_piece()) tc_commit(bars.q_empty());
          }
          if (pend_n >= 0) {   // one pending tile at most: MMA2(n-1) before tile n waits
            ok = do_mma2(pend_n, pend_u, pend_first, pend_last);
            if (!ok) break;
          }
          pend_n = n; pend_u = u; pend_first = first; pend_last = it.last_of_piece();
          if (it.last_of_piece()) ++u;
          it.next();
          ++n;
        }
        if (ok && pend_n >= 0) do_mma2(pend_n, pend_u, pend_first, pend_last);
        // drain: all issued MMAs complete before TMEM is released
        tc_commit(bars.mma_done());
        volatile int never = 0;
        mbar_wait(bars.mma_done(), 0, &never, lim);
      }
    } else if (INT4 && warp >= 2) {
      // ============================================================ dequantisation
      const int tid_dq = threadIdx.x - 64;   // 0..63: token rows tid_dq, tid_dq + 64
      TileIter it;
      it.init(&a.sched, w);
      int n = 0;
      bool ok = true;
      int lo_b = -1, lo = INT_MAX;   // residual window: tokens from lo on may sit in the ring
      while (ok && it.valid()) {
        const int rs = n % a.NRAW, cs = n % a.NC;
        if (RESID && it.b != lo_b) {   // once per sequence, ahead of the stage wait
          lo_b = it.b;
          lo = __ldg(a.seq_lens + it.b) - MLA_RESID_WINDOW;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(bars.raw_full(rs), (n / a.NRAW) & 1, abort_flag, lim));
        if (ok && n >= a.NC)
          ok = __all_sync(0xffffffffu, mbar_wait(bars.c_empty(cs), ((n / a.NC) - 1) & 1, abort_flag, lim));
        if (!ok) break;
        const int nvalid = min(kTile, it.t1 - it.t);
        const uint8_t* raw = sbase + a.off_raw + rs * raw_stage;
        for (int rr = 0; rr < 2; ++rr) {
          const int tok = tid_dq + 64 * rr;
          uint8_t* C = sbase + a.off_c + cs * c_stage + tok * 128;
          const int tp = it.t + tok;
          const size_t rslot = (size_t)it.b * MLA_RESID_WINDOW + (tp & (MLA_RESID_WINDOW - 1));
          if (RESID && tok < nvalid && tp >= lo && __ldg(a.resid_pos + rslot) == tp) {
            const uint4* src = reinterpret_cast<const uint4*>(a.c_resid + rslot * dc);
            for (int half = 0; half < dc / 64; ++half)
  #pragma unroll
              for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4*>(C + half * kBox + ((ch ^ (tok & 7)) * 16)) = __ldg(src + half * 8 + ch);
          } else if (tok < nvalid) {
            const __half* sc = reinterpret_cast<const __half*>(raw + raw_codes) + tok * (dc / 32);
            const uint8_t* codes = raw + tok * (dc / 64) * kCodeBytes64;
            for (int half = 0; half < dc / 64; ++half) {
              const float s0 = __half2float(sc[half * 2]), s1 = __half2float(sc[half * 2 + 1]);
              if (QB == 4) {   // two's-complement nibbles, element 2i in the low nibble of byte i
                const uint4 c0 = *reinterpret_cast<const uint4*>(codes + half * 32);
                const uint4 c1 = *reinterpret_cast<const uint4*>(codes + half * 32 + 16);
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
                  *reinterpret_cast<uint4*>(C + half * kBox + ((ch ^ (tok & 7)) * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
              } else {         // two's-complement 2-bit fields, element 4i+k in bits 2k..2k+1 of byte i
                const uint4 c0 = *reinterpret_cast<const uint4*>(codes + half * 16);
                const uint32_t words[4] = {c0.x, c0.y, c0.z, c0.w};
  #pragma unroll
                for (int ch = 0; ch < 8; ++ch) {           // 8 latent values: 16 bits of codes
                  const uint32_t bits = (words[ch >> 1] >> (16 * (ch & 1))) & 0xFFFFu;
                  const float s = ch < 4 ? s0 : s1;
                  uint32_t o[4];
  #pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    const int f0 = (int)((bits >> (4 * j)) & 3u), f1 = (int)((bits >> (4 * j + 2)) & 3u);
                    o[j] = pack_bf16x2((float)(f0 >= 2 ? f0 - 4 : f0) * s, (float)(f1 >= 2 ? f1 - 4 : f1) * s);
                  }
                  *reinterpret_cast<uint4*>(C + half * kBox + ((ch ^ (tok & 7)) * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
              }
            }
          } else {
            for (int half = 0; half < dc / 64; ++half)
  #pragma unroll
              for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(C + half * kBox + ch * 16) = make_uint4(0, 0, 0, 0);
          }
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
  } else {
    setmaxnreg_inc<224>();
    // ============================================================ softmax + epilogue
    // eight warps: two per TMEM lane quarter (tokens 32q .. 32q+31), each one head half
    const int q = warp & 3;
    const int sw = warp - 4;             // softmax warp 0..7
    const int hh = sw >> 2;              // heads 16hh .. 16hh+15
    const int tr = 32 * q + lane;        // this thread's token row in the tile
    TileIter it;
    it.init(&a.sched, w);
    int n = 0, u = 0, gphase0 = 0, gphase1 = 0;
    bool ok = true;
    float m[kHh], l[kHh];
    auto wwait = [&](uint32_t bar, int parity) -> bool {  // warp-uniform outcome
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, lim));
    };
    auto grp_sync = [&](int i) -> bool {  // all softmax warps, bounded
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.grp(i));
      const int ph = i ? gphase1++ : gphase0++;
      return wwait(bars.grp(i), ph & 1);
    };
    const int G = kH / (R / R2);         // query heads per KV head
    // RoPE keys: a tile's keys (128 token rows of n_kv*2r values) come into the shared stage
    // as 64-column boxes with the 128-byte swizzle: row t of a box holds 8 KV heads' 2r = 8
    // dims, the 16-byte chunk of head g at chunk (g % 8) ^ (t % 8), so a warp whose lane t
    // reads "KV head g of token t" hits 8 different chunks per 8 rows (conflict-free).  Each
    // warp moves its part (its 32 tokens, the KV heads of its 16 heads) into registers as
    // soon as the copy lands and releases the stage; the eighth warp to release it issues
    // the copy of the tile after.  The registers hold tile n+1's keys while tile n is
    // processed, so the copy of tile n+2 has a whole tile period to land.
    const int n_kbox = R / 64;   // 64-column boxes per tile (8 KV heads of 2r = 8 each)
    uint4 kr[kHh];
    auto issue_kr = [&](const TileIter& ti) {   // one thread
      if (!ti.valid()) return;
      const MlaLoc lc = tc_loc<PAGED>(a, ti.b, ti.t);
      const int row = lc.pb * lc.cap + lc.pt;
      fence_proxy_async_smem();
      mbar_expect_tx(bars.kr_full(), (uint32_t)n_kbox * kBox);
      for (int k = 0; k < n_kbox; ++k)
        tma_load_2d(sbase_u32 + a.off_kr + k * kBox, &tm_kr, bars.kr_full(), k * 64, row);
      misc->kr_issued += 1;
    };
    auto fetch_kr = [&](int k, const TileIter& ti_after) -> bool {   // tile k's keys -> kr
      if (!wwait(bars.kr_full(), k & 1)) return false;
      const uint8_t* rowp = sbase + a.off_kr + tr * 128;
#pragma unroll
      for (int h = 0; h < kHh; ++h) {
        const int g = (kHh * hh + h) / G;
        kr[h] = *reinterpret_cast<const uint4*>(rowp + (g >> 3) * kBox + (((g & 7) ^ (tr & 7)) << 4));
      }
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        if (atomicAdd(&misc->kr_released, 1) % kSoftWarps == kSoftWarps - 1) issue_kr(ti_after);
      }
      return true;
    };
    if (it.valid()) {   // a worker with no tiles issues and waits for nothing
      for (int i = threadIdx.x - 128; i < kH * R2; i += 32 * kSoftWarps)
        qr_s[i] = __ldg(a.qrope + (size_t)it.b * kH * R2 + i);
      if (sw == 0 && lane == 0) issue_kr(it);
      TileIter nx = it;
      nx.next();
      ok = fetch_kr(0, nx);
      if (ok) ok = grp_sync(1);   // the first piece's RoPE queries are in place
    }
    while (ok && it.valid()) {
      const int pc = it.pc;
      const bool first = it.first_of_piece();
      if (first) {   // this piece's RoPE queries are in qr_s[u & 1] (loaded one piece ahead)
#pragma unroll
        for (int h = 0; h < kHh; ++h) { m[h] = -INFINITY; l[h] = 0.f; }
      }
      const float* qr = qr_s + (u & 1) * (kH * R2);
      const int sb = n & 1, pb = n % a.NP, ob = u % a.NO;
      const int nvalid = min(kTile, it.t1 - it.t);
      const bool valid = tr < nvalid;
      ok = wwait(bars.s_full(sb), (n >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      float v[kHh];
      {
        uint32_t raw[16];
        tmem_ld16(taddr(tmem, 32 * q, S_COL + sb * kH + kHh * hh), raw);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < kHh; ++h) v[h] = u2f(raw[h]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.s_empty(sb));
      // RoPE score: head 16hh + h against the 2r dims of its KV head
#pragma unroll
      for (int h = 0; h < kHh; ++h) {
        const int H = kHh * hh + h;
        const uint4 kw = kr[h];
        const float4 qa = *reinterpret_cast<const float4*>(qr + H * R2);
        const float4 qb = *reinterpret_cast<const float4*>(qr + H * R2 + 4);
        v[h] += qa.x * bf16lo(kw.x) + qa.y * bf16hi(kw.x) + qa.z * bf16lo(kw.y) + qa.w * bf16hi(kw.y) +
                qb.x * bf16lo(kw.z) + qb.y * bf16hi(kw.z) + qb.z * bf16lo(kw.w) + qb.w * bf16hi(kw.w);
      }
      {
        TileIter nx = it;
        nx.next();
        if (nx.valid()) {
          TileIter nx2 = nx;
          nx2.next();
          ok = fetch_kr(n + 1, nx2);
          if (!ok) break;
        }
      }
      if (!valid) {
#pragma unroll
        for (int h = 0; h < kHh; ++h) v[h] = -INFINITY;
      }
      // per-head maximum over this warp's 32 tokens, published for the other quarters; after
      // the barrier every warp knows the tile's exact per-head maximum, and raises its running
      // max (lazily: only when some score exceeds it by more than tau) identically with the
      // other warps of its head half
      {
        float wmax = -INFINITY;   // lane h ends with head 16hh + h
#pragma unroll
        for (int h = 0; h < kHh; ++h) {
          const float r = warp_max(v[h]);
          wmax = (lane == h) ? r : wmax;
        }
        if (lane < 16) misc->red_max[n & 1][q][kHh * hh + lane] = wmax;
      }
      ok = grp_sync(0);
      if (!ok) break;
      float tmax[kHh];
#pragma unroll
      for (int h4 = 0; h4 < kHh; h4 += 4) {
        const float4 q0 = *reinterpret_cast<const float4*>(&misc->red_max[n & 1][0][kHh * hh + h4]);
        const float4 q1 = *reinterpret_cast<const float4*>(&misc->red_max[n & 1][1][kHh * hh + h4]);
        const float4 q2 = *reinterpret_cast<const float4*>(&misc->red_max[n & 1][2][kHh * hh + h4]);
        const float4 q3 = *reinterpret_cast<const float4*>(&misc->red_max[n & 1][3][kHh * hh + h4]);
        tmax[h4 + 0] = fmaxf(fmaxf(q0.x, q1.x), fmaxf(q2.x, q3.x));
        tmax[h4 + 1] = fmaxf(fmaxf(q0.y, q1.y), fmaxf(q2.y, q3.y));
        tmax[h4 + 2] = fmaxf(fmaxf(q0.z, q1.z), fmaxf(q2.z, q3.z));
        tmax[h4 + 3] = fmaxf(fmaxf(q0.w, q1.w), fmaxf(q2.w, q3.w));
      }
      bool need = false;
#pragma unroll
      for (int h = 0; h < kHh; ++h) need |= (tmax[h] - m[h] > kTau);
      if (need) {
        bool any_scale = false;
        float my_alpha = 1.f;   // the factor of head 16hh + lane (lanes < 16)
#pragma unroll
        for (int h = 0; h < kHh; ++h) {
          const float mn = fmaxf(m[h], tmax[h]);
          const float al = exp2f(m[h] - mn);   // m = -inf on a piece's first tile -> 0
          any_scale |= (mn != m[h]);
          m[h] = mn;
          l[h] *= al;
          if (h == lane) my_alpha = al;
        }
        if (!first && any_scale && q < 2 && hh == q) {
          // O^T rows of heads 16q .. 16q+15 (lanes 0-15 of quarter q) hold the tiles before
          // this one: wait for MMA2(n-1), rescale them in TMEM
          const int pn = n - 1;
          if (!wwait(bars.p_empty(pn % a.NP), (pn / a.NP) & 1)) { ok = false; break; }
          tc_fence_after();
          for (int cc = 0; cc < dc / 16; ++cc) {
            const uint32_t ta = taddr(tmem, 32 * q, O_COL + ob * dc + 16 * cc);
            uint32_t o[16];
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = f2u(u2f(o[k]) * my_alpha);
            tmem_st16(ta, o);
          }
          tmem_wait_st();
        }
      }
      // probabilities of this tile, P^T for MMA2 (row h, column = token, bf16)
      float pr[kHh];
#pragma unroll
      for (int h = 0; h < kHh; ++h) {
        pr[h] = valid ? exp2f(v[h] - m[h]) : 0.f;
        l[h] += pr[h];
      }
      if (n >= a.NP) {
        ok = wwait(bars.p_empty(pb), ((n / a.NP) - 1) & 1);
        if (!ok) break;
      }
      {
        uint8_t* Pt = sbase + a.off_p + pb * kPtBytes + (tr >> 6) * kPtAtom + (tr & 7) * 2;
        const int c8 = (tr & 63) >> 3;
#pragma unroll
        for (int h = 0; h < kHh; ++h) {
          const int H = kHh * hh + h;
          *reinterpret_cast<__nv_bfloat16*>(Pt + H * 128 + ((c8 ^ (H & 7)) << 4)) = __float2bfloat16_rn(pr[h]);
        }
      }
      if (!INT4 && !valid) {
        // rows past the sequence end: clear this token's latent row (both warps of the
        // quarter take half the boxes) so MMA2 never multiplies stale cache contents
        uint8_t* C = sbase + a.off_c + (n % a.NC) * c_stage + tr * 128;
        for (int cb = hh; cb < n_cbox; cb += 2)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(C + cb * kBox + ch * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full(pb));

      if (it.last_of_piece()) {
        // ---------------- piece epilogue: partial (m, l, O) for the split merge
        const float lsum = transpose_reduce16<false>(l, lane);   // l is reset by the next piece
        if (lane < 16) misc->red_l[q][kHh * hh + lane] = lsum;
        {   // the next piece's RoPE queries, into the other buffer (visible after the barrier)
          TileIter nx = it;
          nx.next();
          if (nx.valid())
            for (int i = threadIdx.x - 128; i < kH * R2; i += 32 * kSoftWarps)
              qr_s[((u + 1) & 1) * (kH * R2) + i] = __ldg(a.qrope + (size_t)nx.b * kH * R2 + i);
        }
        ok = grp_sync(1);
        if (!ok) break;
        if (q == 0 && lane < 16) {
          const int H = kHh * hh + lane;
          const float L = misc->red_l[0][H] + misc->red_l[1][H] + misc->red_l[2][H] + misc->red_l[3][H];
          float mh = m[0];
#pragma unroll
          for (int h = 1; h < kHh; ++h) mh = (lane == h) ? m[h] : mh;
          a.mlpart[((size_t)H * a.P + pc) * 2] = mh;
          a.mlpart[((size_t)H * a.P + pc) * 2 + 1] = L;
        }
        ok = wwait(bars.o_full(ob), (u / a.NO) & 1);
        if (!ok) break;
        tc_fence_after();
        if (q < 2) {
          // O^T rows (M = 64 layout): head 16q + lane in lane `lane` (< 16) of quarter q; the
          // two warps of the quarter take one half of the columns each, 32 per TMEM wait
          const int H = 16 * q + lane;
          float* dst = a.opart + ((size_t)pc * kH + H) * dc;
          const int half = dc / 2;   // a multiple of 32
          for (int c0 = hh * half; c0 < (hh + 1) * half; c0 += 32) {
            uint32_t o[2][16];
#pragma unroll
            for (int k = 0; k < 2; ++k) tmem_ld16(taddr(tmem, 32 * q, O_COL + ob * dc + c0 + 16 * k), o[k]);
            tmem_wait_ld();
            if (lane < 16) {
#pragma unroll
              for (int k = 0; k < 2; ++k)
#pragma unroll
                  for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<float4*>(dst + c0 + 16 * k + e) =
                        make_float4(u2f(o[k][e]), u2f(o[k][e + 1]), u2f(o[k][e + 2]), u2f(o[k][e + 3]));
            }
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
    // no RoPE key copy may still be landing when the CTA exits
    if (sw == 0 && lane == 0 && misc->kr_issued > 0) {
      volatile int never = 0;
      mbar_wait(bars.kr_full(), (misc->kr_issued - 1) & 1, &never, lim);
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
  int NC, NRAW, NP, NO;
  uint32_t off_c, off_q, off_p, off_raw, off_qr, off_kr, off_bar, off_misc, total;
};

static TcLayout tc_layout(int dc, int R, int r2, bool int4, int qbits) {
  const uint32_t budget = 232448 - 1024;   // max dynamic smem per block minus alignment slack
  const uint32_t c_stage = (uint32_t)(dc / 64) * kBox;
  const uint32_t raw_stage = (uint32_t)kTile * (dc * qbits / 8) + (uint32_t)kTile * (dc / 16);
  const uint32_t q_bytes = (uint32_t)(dc / 64 > 2 ? dc / 64 - 2 : 0) * kQBox;  // boxes 0-1 sit in P^T padding
  const uint32_t qr_bytes = 2u * kH * r2 * 4;   // two pieces' RoPE queries
  const uint32_t kr_bytes = (uint32_t)kTile * R * 2;
  auto size = [&](int nc, int nraw, int np) {
    uint32_t s = nc * c_stage + q_bytes + np * kPtBytes + kr_bytes;
    s += int4 ? ((nraw * raw_stage + 1023) & ~1023u) : 0;
    s += qr_bytes + 8 * (2 * nc + 2 * nraw + kFixedBars) + sizeof(Misc) + 64 + 1024;
    return s;
  };
  int nc = 2, np = 1, nraw = int4 ? 2 : 0;
  for (int it = 0; it < 16; ++it) {  // deepen the rings while they fit (latent stages first)
    bool grew = false;
    if (nc < 6 && size(nc + 1, nraw, np) <= budget) { ++nc; grew = true; }
    if (np < 2 && size(nc, nraw, np + 1) <= budget) { ++np; grew = true; }
    if (int4 && nraw < 4 && size(nc, nraw + 1, np) <= budget) { ++nraw; grew = true; }
    if (!grew) break;
  }
  TcLayout L{};
  L.NC = nc; L.NRAW = nraw; L.NP = np;
  L.NO = (2 * kH + 2 * dc) <= 512 ? 2 : 1;
  uint32_t o = 0;
  L.off_c = o; o += nc * c_stage;
  L.off_p = o; o += np * kPtBytes;
  L.off_q = o; o += q_bytes;
  L.off_raw = o; o += int4 ? ((nraw * raw_stage + 1023) & ~1023u) : 0;
  L.off_qr = o; o += qr_bytes;
  o = (o + 1023) & ~1023u;   // swizzled TMA boxes
  L.off_kr = o; o += kr_bytes;
  o = (o + 15) & ~15u;
  L.off_bar = o; o += 8 * (2 * nc + 2 * nraw + kFixedBars);
  o = (o + 15) & ~15u;
  L.off_misc = o; o += sizeof(Misc);
  L.total = o + 1024;
  return L;
}

}  // namespace tc
}  // namespace mla

// Shapes the tensor-core kernel covers: bf16, 32 query heads, d_c in {64, 128, 256}, r = 4
// kept pairs per KV head (RoPE width a multiple of 64); the int4 and 2-bit caches with d_c = 128.
bool mla_tc_capable(const mla_plan& p) {
  const mla_config_t& cfg = p.cfg;
  if (cfg.dtype != MLA_BF16 || cfg.n_heads != mla::tc::kH) return false;
  if (cfg.d_c % 64 != 0 || cfg.d_c > 256) return false;
  if (p.R == 0 || p.R % 64 != 0 || 2 * cfg.r_pairs != 8) return false;   // 2r = 8 (r = 4) build
  const bool quant = mla_kind_quant(cfg.cache_kind);
  if (quant && cfg.d_c != 128) return false;
  const mla::tc::TcLayout L =
      mla::tc::tc_layout(cfg.d_c, p.R, 2 * cfg.r_pairs, quant, mla_quant_bits(cfg.cache_kind));
  return L.total <= 232448;
}

// The scale rows of a quantised cache are fetched with 1-D bulk copies, which need an even
// capacity.
bool mla_tc_supported(const mla_plan& p, const mla_cache_t& c) {
  if (!mla_tc_capable(p)) return false;
  if (mla_kind_quant(p.cfg.cache_kind) && c.T_cap % 2 != 0) return false;
  return true;
}

cudaError_t mla_launch_decode_tc(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, int B,
                                 const Sched& sched,
                                 const void* qlat, const float* qrope, float* opart, float* mlpart, int P, int G,
                                 cudaStream_t s) {
  using namespace mla::tc;
  const mla_config_t& cfg = p.cfg;
  const bool int4 = mla_kind_quant(cfg.cache_kind);   // quantised latent: 4- or 2-bit codes
  const int qbits = mla_quant_bits(cfg.cache_kind);
  const int dc = cfg.d_c, R = p.R;
  const int code_row = dc * qbits / 8;   // code bytes per token
  CUtensorMap tm_c, tm_q;
  const uint64_t rows = mla_cache_rows(c);
  bool ok = true;
  if (int4)
    ok &= make_map_2d(&tm_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.c_kv, code_row, rows, code_row, code_row, kTile,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    ok &= make_map_2d(&tm_c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c.c_kv, dc, rows, (uint64_t)dc * 2, 64, kTile,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qlat, dc, (uint64_t)B * kH, (uint64_t)dc * 2, 64, kH,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  CUtensorMap tm_kr;
  ok &= make_map_2d(&tm_kr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c.k_rope, R, rows, (uint64_t)R * 2, 64, kTile,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  const TcLayout L = tc_layout(dc, R, 2 * cfg.r_pairs, int4, qbits);
  TcArgs a;
  a.B = B; a.H = kH; a.d_c = dc; a.R = R; a.r2 = 2 * cfg.r_pairs; a.T_cap = c.T_cap; a.P = P;
  a.sched = sched; a.opart = opart; a.mlpart = mlpart; a.qrope = qrope;
  a.scales = (const __half*)c.c_scales; a.err = p.err;
  a.seq_lens = seq_lens;
  a.cache = c;
  a.c_resid = (const __nv_bfloat16*)c.c_resid;
  a.resid_pos = c.resid_pos;
  a.kr_base = (const uint8_t*)c.k_rope;
  a.c_row = int4 ? (uint32_t)code_row : (uint32_t)dc * 2;
  a.kr_row = (uint32_t)R * 2;
  a.wait_ns = (uint64_t)p.opt_wait_us * 1000u;
  a.skip_tile = p.opt_skip_tile;
  a.NC = L.NC; a.NRAW = L.NRAW; a.NP = L.NP; a.NO = L.NO;
  a.off_c = L.off_c; a.off_q = L.off_q; a.off_p = L.off_p; a.off_raw = L.off_raw;
  a.off_qr = L.off_qr; a.off_kr = L.off_kr; a.off_bar = L.off_bar; a.off_misc = L.off_misc;
  // the RoPE width per KV head is a compile-time constant so the score loop fully unrolls
  // and the per-head registers never move to local memory
  const bool resid = int4 && qbits == 4 && c.c_resid, paged = c.block_table != nullptr;
  auto kern = !int4        ? (paged ? decode_tc_kernel<0, false, true, 8> : decode_tc_kernel<0, false, false, 8>)
              : qbits == 2 ? (paged ? decode_tc_kernel<2, false, true, 8> : decode_tc_kernel<2, false, false, 8>)
              : resid      ? (paged ? decode_tc_kernel<4, true, true, 8> : decode_tc_kernel<4, true, false, 8>)
                           : (paged ? decode_tc_kernel<4, false, true, 8> : decode_tc_kernel<4, false, false, 8>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  // the optional profiling events bracket the launch alone, after all host-side set-up
  if ((e = mla_profile_event(p, kProfAttention, false, s)) != cudaSuccess) return e;
  e = mla_launch_kernel(kern, dim3(G), dim3(384), L.total, s, p.opt_pdl, tm_c, tm_q, tm_kr, a);
  if (e != cudaSuccess) return e;
  if ((e = mla_profile_event(p, kProfAttention, true, s)) != cudaSuccess) return e;
  return cudaSuccess;
}

