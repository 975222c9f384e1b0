// Split-K latent attention on the 5th-generation tensor cores with a (query, head) row per
// softmax thread: the decode (one query per sequence) and many queries per sequence (a
// chunk of new tokens: chunked prefill, drafted tokens to verify), where every query
// attends causally over its sequence's latent cache and the queries of a sequence share
// each cache tile they read.
//
// Paper notes "MHA2MLA" (ACL 2025), §关键设计 and §方法详解/整体框架: the converted layer
// scores all heads against the one shared latent (W_uk absorbed into each query), adds the
// separately computed partial-RoPE term, and takes the probability-weighted latent through
// W_uv; a chunk of a long document's tokens reads the same latent prefix with every query.
//
// A unit of work is (sequence b, block of qper = floor(128 / H) consecutive queries):
// qper * H rows (query j, head h), row = H j + h; a single decode query with more than 32
// heads is a unit of H rows, one with at most 32 heads a unit of the MMA's M = 64 form.
// The units' tokens (up to the block's last query) are laid end to end and split among the
// CTAs like the decode's split-K schedule, in tiles of 64 tokens.  Per tile:
//     S[row][t]   = sum_c Qlat[row][c] * C[t][c]              MMA1  M = 64 or 128, N = 64 tokens
//     S[row][t]  += sum_j Qrope[row][j] * KR[t][g(h)][j]       softmax threads (f32 += bf16 x bf16),
//                                                              or MMA1 over block-diagonal query rows
//     O[row][d]  += sum_t P[row][t] * C[t][d]                  MMA2  N = d_c, K = 64
// with the causal mask t <= position of the row's query.  The transposed orientation gives
// each softmax thread a row (or a quarter of a row's tokens): its running max and sum are
// thread-local.  MMA2 reads the C tile already in shared memory as an MN-major operand, so
// each cache byte is read into the SM once per unit.
//
// Roles: a TMA producer (the unit's Q_lat rows, latent and RoPE-key tiles into two rings),
// a single-thread MMA issuer that owns TMEM, dequantising warps for a quantised cache, and
// softmax warps (placement below).  Every wait is bounded; a timeout sets
// MLA_DEVERR_TIMEOUT, drains the copies in flight and releases TMEM.
#include <cuda.h>

#include "decode_common.cuh"
#include "sm100.cuh"

namespace mla {
namespace chunk {

using namespace sm100;

constexpr int kCT = 64;              // tokens per tile
constexpr uint32_t kTBox = 8192;     // cache box: 64 rows x 128 B
constexpr float kTau = 8.0f;         // lazy-rescale threshold, log2 units
// Row capacity of a unit: 128 (MMA M = 128: a block of queries x heads, or the heads of one
// query when there are more than 32), or 32 (MMA M = 64: the heads of one query, at most
// 32; rows 32..63 of the A operands read the next 4 KB of shared memory, whose values only
// reach output rows nobody reads).  A unit holds qper queries x H heads = rows <= ROWS.
// Warps (a warp reads TMEM lane quarter warp % 4 and issues on scheduler warp % 4).
// 128 rows: the softmax warp of quarter q is warp 4 + q; producer 0, MMA issuer 1,
// dequantisers 2 and 3.  32 rows: only quarters 0 and 1 hold rows (16 each), so warps 0, 1,
// 4 and 5 are the softmax warps, two per quarter, each taking half of every tile's tokens;
// the producer and the issuer sit on warps 2 and 3 and the dequantisers on 6 and 7, off the
// softmax warps' schedulers.
template <int ROWS> struct Geo {
  static constexpr int M = ROWS == 32 ? 64 : 128;   // MMA M
  static constexpr int SW = 4;                       // softmax warps
  static constexpr uint32_t QBOX = ROWS * 128u;      // Q_lat box: ROWS rows x 128 B
  static constexpr uint32_t PBYTES = ROWS * 128u;    // P buffer: ROWS rows x 64 tokens bf16
  static constexpr int PROD = ROWS == 32 ? 2 : 0;    // TMA producer warp
  static constexpr int MMA = ROWS == 32 ? 3 : 1;     // TMEM owner and MMA issuer warp
  static constexpr int DQ = ROWS == 32 ? 6 : 2;      // first dequantising warp
};
// A quantised cache with 32-row units runs 12 warps: four dequantising warps (6, 7, 10, 11,
// on the two schedulers without softmax warps), two threads per token row, each taking
// every other group of 32 values; warps 8 and 9 idle.  Otherwise 8 warps and two
// dequantising warps (DQ, DQ + 1), a thread per token row.
template <int ROWS, int QB> struct Crew {
  static constexpr bool WIDE = ROWS == 32 && QB != 0;
  static constexpr int WARPS = WIDE ? 12 : 8;
  static constexpr int NDQ = WIDE ? 4 : 2;   // dequantising warps
  __device__ static int dq_index(int warp) {   // 0..NDQ-1, or -1
    if (WIDE) return warp == 6 ? 0 : warp == 7 ? 1 : warp == 10 ? 2 : warp == 11 ? 3 : -1;
    return warp == Geo<ROWS>::DQ ? 0 : warp == Geo<ROWS>::DQ + 1 ? 1 : -1;
  }
};
constexpr uint32_t kSCol = 0, kOCol = 128;

struct ChunkArgs {
  int q_chunk, nqb, d_c, R, P, T_cap;
  int H, qper, rows;       // heads, queries per unit, rows per unit (qper * H <= the kernel's ROWS)
  int dcp;                 // d_c rounded up to 64: the TMA boxes zero-fill the columns past d_c
  int rtc;                 // RoPE scores on the tensor cores (block-diagonal query rows in MMA1)
  const __half* scales;    // quantised cache: [rows][d_c/32] fp16 group scales
  uint32_t code_row;       // quantised cache: code bytes per token
  Sched sched;
  const int32_t* seq_lens;
  const float* qrope;      // [B*Q][H][2r], rotated at each query's position, scaled
  float* opart;            // [P][rows][d_c]
  float* mlpart;           // [rows][P][2]
  mla_cache_t cache;
  int32_t* err;
  uint64_t wait_ns;
  int NC, NK, NRAW;        // latent stages, RoPE-key stages, code stages
  uint32_t off_q, off_ar, off_p, off_c, off_k, off_raw, off_bar, off_misc;
  uint32_t c_stage, k_stage, raw_stage;
};

struct Bars {
  uint32_t base;
  int NC, NK, NRAW;
  __device__ uint32_t at(int i) const { return base + 8u * (uint32_t)i; }
  __device__ uint32_t c_full(int s) const { return at(s); }
  __device__ uint32_t c_empty(int s) const { return at(NC + s); }
  __device__ uint32_t k_full(int s) const { return at(2 * NC + s); }
  __device__ uint32_t k_empty(int s) const { return at(2 * NC + NK + s); }
  __device__ uint32_t raw_full(int s) const { return at(2 * NC + 2 * NK + s); }
  __device__ uint32_t raw_empty(int s) const { return at(2 * NC + 2 * NK + NRAW + s); }
  __device__ uint32_t fixed(int i) const { return at(2 * NC + 2 * NK + 2 * NRAW + i); }
  __device__ uint32_t s_full(int i) const { return fixed(i); }
  __device__ uint32_t s_empty(int i) const { return fixed(2 + i); }
  __device__ uint32_t p_full(int i) const { return fixed(4 + i); }
  __device__ uint32_t p_empty(int i) const { return fixed(6 + i); }
  __device__ uint32_t o_full() const { return fixed(8); }
  __device__ uint32_t o_empty() const { return fixed(9); }
  __device__ uint32_t q_full() const { return fixed(10); }
  __device__ uint32_t q_empty() const { return fixed(11); }
  __device__ uint32_t mma_done() const { return fixed(12); }
  // 32-row units: the two softmax warps of a lane quarter exchange row maxima every tile
  // (by tile parity) and row sums every piece
  __device__ uint32_t x_max(int par, int q) const { return fixed(13 + 2 * par + q); }
  __device__ uint32_t x_sum(int q) const { return fixed(17 + q); }
};
constexpr int kFixedBars = 19;
constexpr uint32_t kXchgBytes = 768;   // row maxima [2 parities][2 quarters][2 halves][16], sums [2][2][16]

struct Misc {
  uint32_t tmem_base;
  int abort_flag;
};

struct TileIter {
  const Sched* s;
  int pc, pc_end;
  int v, t0, t1;
  int t;
  __device__ void init(const Sched* sc, int w) {
    s = sc;
    pc = sc->worker_first[w];
    pc_end = sc->worker_first[w + 1];
    t = 0;
    if (pc < pc_end) load();
  }
  __device__ void load() { v = s->piece_b[pc]; t0 = s->piece_t0[pc]; t1 = s->piece_t1[pc]; t = t0; }
  __device__ bool valid() const { return pc < pc_end; }
  __device__ bool first_of_piece() const { return t == t0; }
  __device__ bool last_of_piece() const { return t + kCT >= t1; }
  __device__ void next() {
    t += kCT;
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

// s + sum_j q[j] k[j] with both factors bf16 (q packed in pairs like the keys) and the
// products accumulated in f32 by the mixed-precision FMA (no unpacking of the keys).
__device__ __forceinline__ float rope_dot8_bf16(float s, const uint32_t (&q)[4], uint4 kw) {
  float acc0 = s, acc1 = 0.f;
  const uint32_t w[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    asm("{\n\t.reg .b16 ql, qh, kl, kh;\n\tmov.b32 {ql, qh}, %2;\n\tmov.b32 {kl, kh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, ql, kl, %0;\n\tfma.rn.f32.bf16 %1, qh, kh, %1;\n\t}"
        : "+f"(acc0), "+f"(acc1)
        : "r"(q[i]), "r"(w[i]));
  return acc0 + acc1;
}

// Two's-complement 4-bit code (in the low nibble) to float without a conversion
// instruction: the offset code (n ^ 8) goes into the mantissa of 2^23, whose value then
// exceeds 2^23 + 8 by exactly the code.
__device__ __forceinline__ float nib_to_float(uint32_t n) {
  return __uint_as_float(0x4B000000u | ((n ^ 8u) & 15u)) - 8388616.0f;
}
// The same for a 2-bit code (n ^ 2 is the offset code; 2^23 + 2 its zero).
__device__ __forceinline__ float crumb_to_float(uint32_t n) {
  return __uint_as_float(0x4B000000u | ((n ^ 2u) & 3u)) - 8388610.0f;
}

template <bool PAGED>
__device__ __forceinline__ MlaLoc chunk_loc(const ChunkArgs& a, int b, int t) {
  if (!PAGED) return MlaLoc{b, t, a.T_cap};
  return mla_loc(a.cache, b, t, a.err);
}

// Byte offset of 16-byte chunk `c` of row `r` in a 128-byte-swizzled box of 128-byte rows.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)r * 128u + (uint32_t)(((c ^ r) & 7) << 4); }

// ROWS: rows per unit (see Geo); QB: code width of a quantised latent cache (4 or 2),
// whose rows warps 2-3 dequantise into the latent ring, 0 for a bf16 latent loaded by TMA;
// RESID: the int4 cache's residual window (decode only: the window follows the one query's
// length); PAGED: cache addressed through a block table.
//
// Rings: the latent tile of tile n sits in stage n % NC until MMA2(n) has read it; its RoPE
// keys in stage n % NK, released after MMA1(n) when the RoPE scores run on the tensor cores
// (a.rtc), else after MMA2(n) (the softmax warps read them).
template <int ROWS, int QB, bool RESID, bool PAGED>
__global__ void __launch_bounds__(Crew<ROWS, QB>::WARPS * 32, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_kr,
               const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ ChunkArgs a) {
  constexpr bool QUANT = QB != 0;
  using GG = Geo<ROWS>;
  constexpr int kSW = GG::SW;
  constexpr uint32_t kQBox = GG::QBOX, kPBytes = GG::PBYTES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (sbase_u32 - smem_u32(smem_raw));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int dc = a.d_c, R = a.R, dcp = a.dcp;
  const bool rtc = a.rtc != 0;
  const int n_cbox = dcp / 64, n_kbox = (R + 63) / 64;
  const int kr16 = (R + 15) / 16;   // RoPE K chunks of MMA1 (the boxes zero-fill past R)
  Bars bars{sbase_u32 + a.off_bar, a.NC, a.NK, a.NRAW};
  Misc* misc = reinterpret_cast<Misc*>(sbase + a.off_misc);
  volatile int* abort_flag = &misc->abort_flag;
  const uint64_t lim = a.wait_ns;

  if (threadIdx.x == 0) {
    misc->abort_flag = 0;
    // latent stage: its TMA bytes, or both dequantising warps; RoPE-key stage: its TMA bytes
    for (int s = 0; s < a.NC; ++s) {
      mbar_init(bars.c_full(s), QUANT ? Crew<ROWS, QB>::NDQ : 1);
      mbar_init(bars.c_empty(s), 1);
    }
    // a key stage is free after MMA1 (RoPE scores on the tensor cores) or after every
    // softmax warp has read its keys
    for (int s = 0; s < a.NK; ++s) { mbar_init(bars.k_full(s), 1); mbar_init(bars.k_empty(s), rtc ? 1 : kSW); }
    for (int s = 0; s < a.NRAW; ++s) { mbar_init(bars.raw_full(s), 1); mbar_init(bars.raw_empty(s), Crew<ROWS, QB>::NDQ); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars.s_full(i), 1);
      mbar_init(bars.s_empty(i), kSW);
      mbar_init(bars.p_full(i), kSW);
      mbar_init(bars.p_empty(i), 1);
    }
    mbar_init(bars.o_full(), 1);
    mbar_init(bars.o_empty(), kSW);
    mbar_init(bars.q_full(), rtc ? 1 + kSW : 1);   // Q_lat bytes (+ the softmax warps' RoPE rows)
    mbar_init(bars.q_empty(), 1);
    mbar_init(bars.mma_done(), 1);
    for (int i = 0; i < 4; ++i) mbar_init(bars.x_max(i >> 1, i & 1), 2);
    for (int i = 0; i < 2; ++i) mbar_init(bars.x_sum(i), 2);
    fence_mbar_init();
  }
  if (rtc) {   // block-diagonal RoPE query rows: zero once, each piece rewrites one chunk per row
    uint4* ar = reinterpret_cast<uint4*>(sbase + a.off_ar);
    for (int i = threadIdx.x; i < n_kbox * (int)kQBox / 16; i += blockDim.x) ar[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == GG::PROD && lane == 0) {
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_kr);
    tma_prefetch_desc(&tm_q);
  }
  constexpr uint32_t kTmemCols = 512;   // S 2 x 64 columns, O d_c <= 256 columns
  if (warp == GG::MMA) {
    tmem_alloc(smem_u32(&misc->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();   // schedule, absorbed queries and the cache come from earlier kernels
  pdl_trigger();
  const uint32_t tmem = misc->tmem_base;
  const int w = blockIdx.x;
  auto qrow0 = [&](int v) {   // first Q_lat row of unit v: query (v % nqb) * qper of sequence v / nqb
    return ((v / a.nqb) * a.q_chunk + (v % a.nqb) * a.qper) * a.H;
  };

  if (warp == GG::PROD) {
    // ============================================================ TMA producer (lane 0)
    if (lane == 0) {
      // Two cursors over the CTA's tiles: the latent (or code) ring with the query boxes, and
      // the RoPE-key ring, whose stages free up at different times; each copy is issued as
      // soon as its stage is free.
      TileIter ic, ik;
      ic.init(&a.sched, w);
      ik = ic;
      int nc = 0, nk = 0, u = 0, q_loads = 0;
      bool ok = true;
      uint64_t t_idle = globaltimer();
      while (ic.valid() || ik.valid()) {
        bool progress = false;
        if (ic.valid()) {
          const int cs = nc % a.NC, rs = QUANT ? nc % a.NRAW : 0;
          const bool q_ok = !ic.first_of_piece() || u == 0 || mbar_test(bars.q_empty(), (u - 1) & 1);
          const bool slot_ok = QUANT ? (nc < a.NRAW || mbar_test(bars.raw_empty(rs), ((nc / a.NRAW) - 1) & 1))
                                     : (nc < a.NC || mbar_test(bars.c_empty(cs), ((nc / a.NC) - 1) & 1));
          if (q_ok && slot_ok) {
            if (ic.first_of_piece()) {
              mbar_expect_tx(bars.q_full(), (uint32_t)n_cbox * kQBox);
              for (int kb = 0; kb < n_cbox; ++kb)
                tma_load_2d(sbase_u32 + a.off_q + kb * kQBox, &tm_q, bars.q_full(), kb * 64, qrow0(ic.v));
              ++q_loads;
            }
            const MlaLoc lc = chunk_loc<PAGED>(a, ic.v / a.nqb, ic.t);   // a 64-token tile lies in one block
            const int row = lc.pb * lc.cap + lc.pt;
            if (!QUANT) {   // latent boxes
              const uint32_t st = sbase_u32 + a.off_c + cs * a.c_stage;
              mbar_expect_tx(bars.c_full(cs), (uint32_t)n_cbox * kTBox);
              for (int kb = 0; kb < n_cbox; ++kb) tma_load_2d(st + kb * kTBox, &tm_c, bars.c_full(cs), kb * 64, row);
            } else {        // code rows (one box of 64 rows) into the raw ring
              const uint32_t rb = sbase_u32 + a.off_raw + rs * a.raw_stage;
              mbar_expect_tx(bars.raw_full(rs), (uint32_t)kCT * a.code_row);
              tma_load_2d(rb, &tm_c, bars.raw_full(rs), 0, row);
            }
            if (ic.last_of_piece()) ++u;
            ic.next();
            ++nc;
            progress = true;
          }
        }
        if (ik.valid() && nk < nc) {   // keys never run ahead of their tile's latent copy
          const int ks = nk % a.NK;
          if (nk < a.NK || mbar_test(bars.k_empty(ks), ((nk / a.NK) - 1) & 1)) {
            const MlaLoc lc = chunk_loc<PAGED>(a, ik.v / a.nqb, ik.t);
            const int row = lc.pb * lc.cap + lc.pt;
            const uint32_t st = sbase_u32 + a.off_k + ks * a.k_stage;
            mbar_expect_tx(bars.k_full(ks), (uint32_t)n_kbox * kTBox);
            for (int kb = 0; kb < n_kbox; ++kb) tma_load_2d(st + kb * kTBox, &tm_kr, bars.k_full(ks), kb * 64, row);
            ik.next();
            ++nk;
            progress = true;
          }
        }
        if (progress) {
          t_idle = globaltimer();
        } else {
          if (*abort_flag || globaltimer() - t_idle > lim) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          __nanosleep(32);
        }
      }
      (void)ok;
      // drain: every issued copy lands before the CTA exits (copies not issued because the
      // wait gave up are not waited for)
      volatile int never = 0;
      if (q_loads > 0) mbar_wait(bars.q_full(), (q_loads - 1) & 1, &never, lim);
      auto drain = [&](int NS, int issued, auto bar) {
        const int last = issued - 1;
        for (int s = 0; s < NS; ++s) {
          const int k = last - ((last - s) % NS + NS) % NS;
          if (last >= 0 && k >= 0) mbar_wait(bar(s), (k / NS) & 1, &never, lim);
        }
      };
      if (!QUANT) drain(a.NC, nc, [&](int s) { return bars.c_full(s); });
      else drain(a.NRAW, nc, [&](int s) { return bars.raw_full(s); });
      drain(a.NK, nk, [&](int s) { return bars.k_full(s); });
    }
  } else if (warp == GG::MMA) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = idesc_bf16_f32(GG::M, kCT, false, false);   // S[row][t]
      const uint32_t idesc2 = idesc_bf16_f32(GG::M, dcp, false, true);    // O[row][d]
      TileIter it;
      it.init(&a.sched, w);
      int n = 0, u = 0;
      bool ok = true;
      int pend_n = -1, pend_u = 0;
      bool pend_first = false, pend_last = false;
      auto do_mma2 = [&](int pn, int pu, bool first, bool lastp) -> bool {
        const int pb = pn & 1, cs = pn % a.NC;
        if (!mbar_wait(bars.p_full(pb), (pn >> 1) & 1, abort_flag, lim)) return false;
        if (first && pu > 0)
          if (!mbar_wait(bars.o_empty(), (pu - 1) & 1, abort_flag, lim)) return false;
        tc_fence_after();
        const uint32_t c0 = sbase_u32 + a.off_c + cs * a.c_stage;
        const uint32_t p0 = sbase_u32 + a.off_p + pb * kPBytes;
#pragma unroll
        for (int kk = 0; kk < kCT / 16; ++kk) {
          const uint64_t ad = smem_desc(p0 + kk * 32, 16, 1024, kLayoutSW128);
          const uint64_t bd = smem_desc(c0 + kk * 2048, kTBox, 1024, kLayoutSW128);
          tc_mma_bf16(tmem + kOCol, ad, bd, idesc2, (first && kk == 0) ? 0u : 1u);
        }
        tc_commit(bars.p_empty(pb));
        tc_commit(bars.c_empty(cs));
        if (lastp) tc_commit(bars.o_full());
        return true;
      };
      while (ok && it.valid()) {
        const int sb = n & 1, cs = n % a.NC, ks = n % a.NK;
        const bool first = it.first_of_piece();
        {
          const uint64_t t_start = globaltimer();
          while (true) {
            if (pend_n >= 0 && mbar_test(bars.p_full(pend_n & 1), (pend_n >> 1) & 1)) {
              ok = do_mma2(pend_n, pend_u, pend_first, pend_last);
              pend_n = -1;
              if (!ok) break;
              continue;
            }
            if ((n < 2 || mbar_test(bars.s_empty(sb), ((n >> 1) - 1) & 1)) &&
                (!first || mbar_test(bars.q_full(), u & 1)) && mbar_test(bars.c_full(cs), (n / a.NC) & 1) &&
                (!rtc || mbar_test(bars.k_full(ks), (n / a.NK) & 1)))   // MMA1 reads keys only with rtc
              break;
            if (*abort_flag || globaltimer() - t_start > lim) {
              *abort_flag = 1;
              ok = false;
              break;
            }
            __nanosleep(32);   // leave the scheduler's issue slots to the other warps
          }
        }
        if (!ok) break;
        tc_fence_after();
        {  // MMA1: S = Q_lat C^T (+ Q_rope KR^T)
          const uint32_t c0 = sbase_u32 + a.off_c + cs * a.c_stage;
          const uint32_t d = tmem + kSCol + sb * kCT;
          for (int kk = 0; kk < dcp / 16; ++kk) {
            const uint64_t ad = smem_desc(sbase_u32 + a.off_q + (kk >> 2) * kQBox + (kk & 3) * 32, 16, 1024,
                                          kLayoutSW128);
            const uint64_t bd = smem_desc(c0 + (kk >> 2) * kTBox + (kk & 3) * 32, 16, 1024, kLayoutSW128);
            tc_mma_bf16(d, ad, bd, idesc1, kk > 0 ? 1u : 0u);
          }
          if (rtc) {
            const uint32_t k0 = sbase_u32 + a.off_k + ks * a.k_stage;
            for (int kk = 0; kk < kr16; ++kk) {
              const uint64_t ad = smem_desc(sbase_u32 + a.off_ar + (kk >> 2) * kQBox + (kk & 3) * 32, 16, 1024,
                                            kLayoutSW128);
              const uint64_t bd = smem_desc(k0 + (kk >> 2) * kTBox + (kk & 3) * 32, 16, 1024, kLayoutSW128);
              tc_mma_bf16(d, ad, bd, idesc1, 1u);
            }
            tc_commit(bars.k_empty(ks));
          }
          tc_commit(bars.s_full(sb));
          if (it.last_of_piece()) tc_commit(bars.q_empty());
        }
        if (pend_n >= 0) {
          ok = do_mma2(pend_n, pend_u, pend_first, pend_last);
          if (!ok) break;
        }
        pend_n = n; pend_u = u; pend_first = first; pend_last = it.last_of_piece();
        if (it.last_of_piece()) ++u;
        it.next();
        ++n;
      }
      if (ok && pend_n >= 0) do_mma2(pend_n, pend_u, pend_first, pend_last);
      tc_commit(bars.mma_done());
      volatile int never = 0;
      mbar_wait(bars.mma_done(), 0, &never, lim);
    }
  } else if (QUANT && Crew<ROWS, QB>::dq_index(warp) >= 0) {
    // ============================================================ dequantisation
    // thread = token row of the tile (with four dequantising warps: a token row and the
    // groups of one parity): codes * scale -> bf16 into the latent stage's swizzled boxes;
    // rows past the unit's last token are zeroed (MMA2 multiplies them by P = 0)
    constexpr int NPART = Crew<ROWS, QB>::NDQ / 2;   // threads per token row
    const int dqt = Crew<ROWS, QB>::dq_index(warp) * 32 + lane;
    const int tok = dqt & 63, part = dqt >> 6;        // token row, group parity (NPART = 2)
    TileIter it;
    it.init(&a.sched, w);
    int n = 0;
    bool ok = true;
    int lo_v = -1, lo = INT_MAX;   // residual window (decode): tokens from lo on may sit in the ring
    // this token's group scales (up to 8 per token) come from global memory with plain loads,
    // issued two tiles ahead so their latency hides behind the dequantisation of two tiles
    auto load_scales = [&](const TileIter& ti, __half (&sc)[8]) {
#pragma unroll
      for (int j = 0; j < 8; ++j) sc[j] = __float2half(0.f);
      if (!ti.valid() || tok >= ti.t1 - ti.t) return;
      const MlaLoc lc = chunk_loc<PAGED>(a, ti.v / a.nqb, ti.t);
      const __half* sp = a.scales + ((size_t)lc.pb * lc.cap + lc.pt + tok) * (dc / 32);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < dc / 32) sc[j] = __ldg(sp + j);
    };
    TileIter pf = it;
    __half scl[8], scl1[8], scl2[8];   // tiles n, n + 1, n + 2
    load_scales(pf, scl);
    if (pf.valid()) pf.next();
    load_scales(pf, scl1);
    if (pf.valid()) pf.next();
    load_scales(pf, scl2);
    while (ok && it.valid()) {
      const int rs = n % a.NRAW, cs = n % a.NC;
      if (RESID && it.v != lo_v) {   // once per sequence, ahead of the stage wait
        lo_v = it.v;
        lo = __ldg(a.seq_lens + it.v) - MLA_RESID_WINDOW;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bars.raw_full(rs), (n / a.NRAW) & 1, abort_flag, lim));
      if (ok && n >= a.NC)
        ok = __all_sync(0xffffffffu, mbar_wait(bars.c_empty(cs), ((n / a.NC) - 1) & 1, abort_flag, lim));
      if (!ok) break;
      const int nvalid = min(kCT, it.t1 - it.t);
      const uint8_t* raw = sbase + a.off_raw + rs * a.raw_stage;
      uint8_t* C = sbase + a.off_c + cs * a.c_stage;
      const int tp = it.t + tok;
      const size_t rslot = (size_t)it.v * MLA_RESID_WINDOW + (tp & (MLA_RESID_WINDOW - 1));
      // latent value j of the row goes to box j / 64, 16-byte chunk (j % 64) / 8 (swizzled)
      auto put = [&](int chunk, uint4 v) {
        *reinterpret_cast<uint4*>(C + (chunk >> 3) * kTBox + sw128(tok, chunk)) = v;
      };
      if (RESID && tok < nvalid && tp >= lo && __ldg(a.cache.resid_pos + rslot) == tp) {
        // one of the window's tokens: its unquantised row from the ring
        const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.cache.c_resid) +
                                                          rslot * dc);
        for (int j = part; j < dc / 8; j += NPART) put(j, __ldg(src + j));
      } else if (tok < nvalid) {
        const uint8_t* codes = raw + tok * a.code_row;
        float svs[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) svs[j] = __half2float(scl[j]);
#pragma unroll 1
        for (int grp = part; grp < dc / 32; grp += NPART) {   // 32 values, one scale (a loop: code size)
          float sv = svs[0];
#pragma unroll
          for (int j = 1; j < 8; ++j) sv = grp == j ? svs[j] : sv;
          if (QB == 4) {   // two's-complement nibbles, element 2i in the low nibble of byte i
            const uint4 cw = *reinterpret_cast<const uint4*>(codes + grp * 16);
            const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t o[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t byte = (words[ch] >> (8 * j)) & 0xFFu;
                o[j] = pack_bf16x2(nib_to_float(byte) * sv, nib_to_float(byte >> 4) * sv);
              }
              put(grp * 4 + ch, make_uint4(o[0], o[1], o[2], o[3]));
            }
          } else {         // two's-complement 2-bit fields, element 4i+k in bits 2k..2k+1 of byte i
            const uint2 cw = *reinterpret_cast<const uint2*>(codes + grp * 8);
            const uint32_t words[2] = {cw.x, cw.y};
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              const uint32_t bits = (words[ch >> 1] >> (16 * (ch & 1))) & 0xFFFFu;
              uint32_t o[4];
#pragma unroll
              for (int j = 0; j < 4; ++j)
                o[j] = pack_bf16x2(crumb_to_float(bits >> (4 * j)) * sv, crumb_to_float(bits >> (4 * j + 2)) * sv);
              put(grp * 4 + ch, make_uint4(o[0], o[1], o[2], o[3]));
            }
          }
        }
      } else {
        for (int j = part; j < dc / 8; j += NPART) put(j, make_uint4(0, 0, 0, 0));
      }
      for (int j = dc / 8 + part; j < dcp / 8; j += NPART) put(j, make_uint4(0, 0, 0, 0));   // padding columns
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bars.raw_empty(rs));
        mbar_arrive(bars.c_full(cs));
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) { scl[j] = scl1[j]; scl1[j] = scl2[j]; }
      if (pf.valid()) pf.next();
      load_scales(pf, scl2);
      it.next();
      ++n;
    }
  } else if (ROWS == 32 && (warp & 2) == 0 && warp < 8) {
    // ============================================================ softmax + epilogue, 32 rows
    // Rows 16q .. 16q+15 sit in TMEM lanes 0..15 of quarter q = warp & 1 (M = 64).  Four
    // threads share a row: warp half = warp >> 2 and lane half hb = lane >> 4 take tokens
    // 32 hb + 16 half + [0, 16) of each tile (one 16x32bx2 TMEM load).  The row's running
    // max is common to the four (a shuffle, then an exchange with the other warp of the
    // quarter through shared memory); each keeps its own partial sum.
    const int q = warp & 1, half = warp >> 2, hb = lane >> 4;
    const int r = 16 * q + (lane & 15);
    const int tb = 32 * hb + 16 * half;          // this thread's first token of a tile
    const int sidx = 64 * half + 32 * q + lane;  // 0..127 over the four warps
    const bool valid_row = r < a.rows;
    const int hd = r % a.H;
    const int n_kv = R / 8;
    const int g = hd / (a.H / n_kv);
    float* xmax = reinterpret_cast<float*>(sbase + a.off_misc + 16);   // [2][2][2][16]
    float* xsum = xmax + 128;                                           // [2][2][16]
    TileIter it;
    it.init(&a.sched, w);
    int n = 0, u = 0;
    bool ok = true;
    float m = -INFINITY, l = 0.f;
    float qr[8];
    uint32_t qb[4];   // the RoPE query rounded to bf16, in pairs
    int p_row = -1;
    auto wwait = [&](uint32_t bar, int parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, lim));
    };
    while (ok && it.valid()) {
      const bool first = it.first_of_piece();
      const int pc = it.pc;
      if (first) {
        const int bseq = it.v / a.nqb, i = (it.v % a.nqb) * a.qper + r / a.H;
        p_row = -1;
#pragma unroll
        for (int j = 0; j < 8; ++j) qr[j] = 0.f;
        if (r < a.rows && i < a.q_chunk) {
          p_row = __ldg(a.seq_lens + bseq) - a.q_chunk + i;
          const float4* src = reinterpret_cast<const float4*>(a.qrope + (((size_t)bseq * a.q_chunk + i) * a.H + hd) * 8);
          const float4 x0 = __ldg(src), x1 = __ldg(src + 1);
          qr[0] = x0.x; qr[1] = x0.y; qr[2] = x0.z; qr[3] = x0.w;
          qr[4] = x1.x; qr[5] = x1.y; qr[6] = x1.z; qr[7] = x1.w;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) qb[j] = pack_bf16x2(qr[2 * j], qr[2 * j + 1]);
        m = -INFINITY;
        l = 0.f;
      }
      const int sb = n & 1, pb = n & 1, ks = n % a.NK;
      ok = wwait(bars.s_full(sb), (n >> 1) & 1);
      if (ok) ok = wwait(bars.k_full(ks), (n / a.NK) & 1);   // the RoPE keys of this tile
      if (!ok) break;
      tc_fence_after();
      float s[16];
      {
        uint32_t raw[16];
        tmem_ld16x2<32>(taddr(tmem, 32 * q, kSCol + sb * kCT + 16 * half), raw);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          asm volatile("" : "+r"(raw[e]));   // the values exist only after the wait
          s[e] = u2f(raw[e]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.s_empty(sb));
      // RoPE score against the tile's keys: row tt of the swizzled key stage, KV head g's chunk
      const uint8_t* krb = sbase + a.off_k + ks * a.k_stage + (g >> 3) * kTBox;
      const int lim_t = min(it.t1, p_row + 1) - it.t;   // tokens [0, lim_t) of the tile count
      float mx = -INFINITY;
      {
        uint4 kw[16];   // all 16 keys in flight before the first use
#pragma unroll
        for (int t = 0; t < 16; ++t) kw[t] = *reinterpret_cast<const uint4*>(krb + sw128(tb + t, g));
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.k_empty(ks));   // the keys are in registers
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int tt = tb + t;
          float v = rope_dot8_bf16(s[t], qb, kw[t]);
          v = tt < lim_t ? v : -INFINITY;
          s[t] = v;
          mx = fmaxf(mx, v);
        }
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      {   // the other warp of this quarter holds the row's other 32 tokens
        float* xm = xmax + (((n & 1) * 2 + q) * 2) * 16;
        if (lane < 16) xm[half * 16 + lane] = mx;
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.x_max(n & 1, q));
        if (!wwait(bars.x_max(n & 1, q), (n >> 1) & 1)) { ok = false; break; }
        mx = fmaxf(mx, xm[(1 - half) * 16 + (lane & 15)]);
      }
      // Raise the running max lazily (the four threads of a row decide alike): the TMEM
      // loads and stores are warp-collective, so the warp rescales when any row needs it.
      // Each warp rescales its half of O's columns; lanes 16-31 touch lanes M = 64 leaves unused.
      const bool raise = mx > m + kTau;
      if (__any_sync(0xffffffffu, raise)) {
        const float al = raise ? exp2f(m - mx) : 1.f;   // m = -inf: 0
        if (!first) {
          const int pn = n - 1;
          if (!wwait(bars.p_empty(pn & 1), (pn >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          for (int cc = 0; cc < dcp / 32; ++cc) {
            const uint32_t ta = taddr(tmem, 32 * q, kOCol + half * (dcp / 2) + 16 * cc);
            uint32_t o[16];
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = f2u(u2f(o[k]) * al);
            tmem_st16(ta, o);
          }
          tmem_wait_st();
        }
        if (raise) {
          l *= al;
          m = mx;
        }
      }
      uint32_t pk[8];
      const float mb = m == -INFINITY ? 0.f : m;   // masked scores are -inf: 2^(-inf) = 0
#pragma unroll
      for (int t = 0; t < 16; t += 2) {
        const float p0 = ex2_approx(s[t] - mb), p1 = ex2_approx(s[t + 1] - mb);
        l += p0 + p1;
        pk[t / 2] = pack_bf16x2(p0, p1);
      }
      if (!QUANT && it.t1 - it.t < kCT) {
        // latent rows past the unit's last token (stale cache rows, possibly not finite):
        // zeroed before MMA2 multiplies them by P = 0 (MMA1 has read the stage: S is full)
        const int nvalid = it.t1 - it.t;
        uint8_t* C = sbase + a.off_c + (n % a.NC) * a.c_stage;
        const int nchunk = (kCT - nvalid) * 8 * n_cbox;   // 16-byte chunks
        for (int i = sidx; i < nchunk; i += 128) {
          const int box = i / ((kCT - nvalid) * 8), rem = i % ((kCT - nvalid) * 8);
          *reinterpret_cast<uint4*>(C + box * kTBox + (nvalid + rem / 8) * 128 + (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      if (n >= 2) {
        ok = wwait(bars.p_empty(pb), ((n >> 1) - 1) & 1);
        if (!ok) break;
      }
      {  // P row r, this thread's 16 tokens: chunks tb / 8 and tb / 8 + 1
        uint8_t* prow = sbase + a.off_p + pb * kPBytes;
        *reinterpret_cast<uint4*>(prow + sw128(r, tb / 8)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(prow + sw128(r, tb / 8 + 1)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full(pb));

      if (it.last_of_piece()) {
        // ---------------- piece epilogue: the row's partial (m, l, O)
        float lr = l + __shfl_xor_sync(0xffffffffu, l, 16);
        {
          float* xs = xsum + (q * 2) * 16;
          if (lane < 16) xs[half * 16 + lane] = lr;
          __syncwarp();
          if (lane == 0) mbar_arrive(bars.x_sum(q));
          if (!wwait(bars.x_sum(q), u & 1)) { ok = false; break; }
          lr += xs[(1 - half) * 16 + (lane & 15)];
        }
        if (valid_row && half == 0 && hb == 0) {
          a.mlpart[((size_t)r * a.P + pc) * 2] = m;
          a.mlpart[((size_t)r * a.P + pc) * 2 + 1] = lr;
        }
        ok = wwait(bars.o_full(), u & 1);
        if (!ok) break;
        tc_fence_after();
        // this warp's half of the columns; lanes 16-31 read lanes M = 64 leaves unused
        float* dst = a.opart + ((size_t)pc * a.rows + (valid_row ? r : 0)) * dc;
        for (int c0 = half * (dc / 2); c0 < (half + 1) * (dc / 2); c0 += 16) {
          uint32_t o[16];
          tmem_ld16(taddr(tmem, 32 * q, kOCol + c0), o);
          tmem_wait_ld();
          if (!valid_row || hb) continue;
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(dst + c0 + e) = make_float4(u2f(o[e]), u2f(o[e + 1]), u2f(o[e + 2]), u2f(o[e + 3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.o_empty());
        ++u;
      }
      it.next();
      ++n;
    }
  } else if (ROWS == 128 && warp >= 4) {
    // ============================================================ softmax + epilogue, 128 rows
    // Warp 4 + q reads TMEM lane quarter q = rows 32q .. 32q+31, a row per thread.
    const int q = warp - 4;
    const int r = 32 * q + lane;   // this thread's row
    constexpr int TPL = kCT;       // tokens per thread
    const bool valid_row = r < a.rows;
    const int hd = r % a.H;                  // its head; its query is r / H of the unit
    const int n_kv = R / 8;
    const int g = hd / (a.H / n_kv);         // KV head of this row's head
    TileIter it;
    it.init(&a.sched, w);
    int n = 0, u = 0;
    bool ok = true;
    float m = -INFINITY, l = 0.f;
    float qr[8];
    uint32_t qb[4];   // the RoPE query rounded to bf16, in pairs
    int p_row = -1;                          // position of this row's query (-1: past the chunk)
    auto wwait = [&](uint32_t bar, int parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, lim));
    };
    while (ok && it.valid()) {
      const bool first = it.first_of_piece();
      const int pc = it.pc;
      if (first) {
        const int bseq = it.v / a.nqb, i = (it.v % a.nqb) * a.qper + r / a.H;
        p_row = -1;
#pragma unroll
        for (int j = 0; j < 8; ++j) qr[j] = 0.f;
        if (r < a.rows && i < a.q_chunk) {
          p_row = __ldg(a.seq_lens + bseq) - a.q_chunk + i;
          const float4* src = reinterpret_cast<const float4*>(a.qrope + (((size_t)bseq * a.q_chunk + i) * a.H + hd) * 8);
          const float4 x0 = __ldg(src), x1 = __ldg(src + 1);
          qr[0] = x0.x; qr[1] = x0.y; qr[2] = x0.z; qr[3] = x0.w;
          qr[4] = x1.x; qr[5] = x1.y; qr[6] = x1.z; qr[7] = x1.w;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) qb[j] = pack_bf16x2(qr[2 * j], qr[2 * j + 1]);
        if (rtc) {
          // this row's RoPE query (bf16) into its KV head's 16-byte chunk of the block-diagonal
          // operand, once MMA1 of the previous piece has read it
          if (u > 0 && !wwait(bars.q_empty(), (u - 1) & 1)) { ok = false; break; }
          if (valid_row)
            *reinterpret_cast<uint4*>(sbase + a.off_ar + (g >> 3) * kQBox + sw128(r, g & 7)) =
                make_uint4(pack_bf16x2(qr[0], qr[1]), pack_bf16x2(qr[2], qr[3]), pack_bf16x2(qr[4], qr[5]),
                           pack_bf16x2(qr[6], qr[7]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bars.q_full());
        }
        m = -INFINITY;
        l = 0.f;
      }
      const int sb = n & 1, pb = n & 1, ks = n % a.NK;
      ok = wwait(bars.s_full(sb), (n >> 1) & 1);
      if (ok && !rtc) ok = wwait(bars.k_full(ks), (n / a.NK) & 1);   // the RoPE keys of this tile
      if (!ok) break;
      tc_fence_after();
      float s[kCT];
      {
        uint32_t raw[kCT];
#pragma unroll
        for (int k = 0; k < kCT / 16; ++k)
          tmem_ld16(taddr(tmem, 32 * q, kSCol + sb * kCT + 16 * k), *reinterpret_cast<uint32_t(*)[16]>(raw + 16 * k));
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < kCT; ++e) {
          asm volatile("" : "+r"(raw[e]));   // the values exist only after the wait
          s[e] = u2f(raw[e]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.s_empty(sb));
      const int lim_t = min(it.t1, p_row + 1) - it.t;   // tokens [0, lim_t) of the tile count
      float mx = -INFINITY;
      if (rtc) {
#pragma unroll
        for (int t = 0; t < TPL; ++t) {
          const float v = t < lim_t ? s[t] : -INFINITY;
          s[t] = v;
          mx = fmaxf(mx, v);
        }
      } else {
        // RoPE score against the tile's keys: row tt of the swizzled stage, KV head g's chunk
        const uint8_t* krb = sbase + a.off_k + ks * a.k_stage + (g >> 3) * kTBox;
#pragma unroll
        for (int t0 = 0; t0 < TPL; t0 += 16) {   // 16 keys in flight at a time
          uint4 kw[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) kw[t] = *reinterpret_cast<const uint4*>(krb + sw128(t0 + t, g));
          if (t0 + 16 == TPL) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.k_empty(ks));   // this warp holds all its keys
          }
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int tt = t0 + t;
            float v = rope_dot8_bf16(s[tt], qb, kw[t]);
            v = tt < lim_t ? v : -INFINITY;
            s[tt] = v;
            mx = fmaxf(mx, v);
          }
        }
      }
      // Raise the running max lazily: a row rescales when its max grew by more than kTau.
      // Rows decide on their own, but the TMEM loads and stores (and the wait before them)
      // are warp-collective, so the warp takes the branch when any of its rows needs it and
      // the other rows multiply by 1.
      const bool raise = mx > m + kTau;
      if (__any_sync(0xffffffffu, raise)) {
        const float al = raise ? exp2f(m - mx) : 1.f;   // m = -inf: 0
        if (!first) {
          // O holds the piece's tiles before this one: wait for MMA2(n-1), then rescale
          const int pn = n - 1;
          if (!wwait(bars.p_empty(pn & 1), (pn >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          for (int cc = 0; cc < dcp / 16; ++cc) {
            const uint32_t ta = taddr(tmem, 32 * q, kOCol + 16 * cc);
            uint32_t o[16];
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = f2u(u2f(o[k]) * al);
            tmem_st16(ta, o);
          }
          tmem_wait_st();
        }
        if (raise) {
          l *= al;
          m = mx;
        }
      }
      uint32_t pk[TPL / 2];
      const float mb = m == -INFINITY ? 0.f : m;   // masked scores are -inf: 2^(-inf) = 0
#pragma unroll
      for (int t = 0; t < TPL; t += 2) {
        const float p0 = ex2_approx(s[t] - mb), p1 = ex2_approx(s[t + 1] - mb);
        l += p0 + p1;
        pk[t / 2] = pack_bf16x2(p0, p1);
      }
      if (!QUANT && it.t1 - it.t < kCT) {
        // latent rows past the unit's last token (stale cache rows, possibly not finite):
        // zeroed before MMA2 multiplies them by P = 0 (MMA1 has read the stage: S is full)
        const int nvalid = it.t1 - it.t;
        uint8_t* C = sbase + a.off_c + (n % a.NC) * a.c_stage;
        const int nchunk = (kCT - nvalid) * 8 * n_cbox;   // 16-byte chunks
        for (int i = r; i < nchunk; i += ROWS) {
          const int box = i / ((kCT - nvalid) * 8), rem = i % ((kCT - nvalid) * 8);
          *reinterpret_cast<uint4*>(C + box * kTBox + (nvalid + rem / 8) * 128 + (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      if (n >= 2) {
        ok = wwait(bars.p_empty(pb), ((n >> 1) - 1) & 1);
        if (!ok) break;
      }
      {  // P row r: 64 tokens = 128 B, 16-byte chunk c at (c ^ (r % 8))
        uint8_t* prow = sbase + a.off_p + pb * kPBytes;
#pragma unroll
        for (int c = 0; c < TPL / 8; ++c)
          *reinterpret_cast<uint4*>(prow + sw128(r, c)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full(pb));

      if (it.last_of_piece()) {
        // ---------------- piece epilogue: this row's partial (m, l, O)
        if (valid_row) {
          a.mlpart[((size_t)r * a.P + pc) * 2] = m;
          a.mlpart[((size_t)r * a.P + pc) * 2 + 1] = l;
        }
        ok = wwait(bars.o_full(), u & 1);
        if (!ok) break;
        tc_fence_after();
        float* dst = a.opart + ((size_t)pc * a.rows + (valid_row ? r : 0)) * dc;
        for (int c0 = 0; c0 < dc; c0 += 32) {
          uint32_t o[2][16];
#pragma unroll
          for (int k = 0; k < 2; ++k) tmem_ld16(taddr(tmem, 32 * q, kOCol + c0 + 16 * k), o[k]);
          tmem_wait_ld();
          if (!valid_row) continue;
#pragma unroll
          for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              *reinterpret_cast<float4*>(dst + c0 + 16 * k + e) =
                  make_float4(u2f(o[k][e]), u2f(o[k][e + 1]), u2f(o[k][e + 2]), u2f(o[k][e + 3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.o_empty());
        ++u;
      }
      it.next();
      ++n;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == GG::MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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

// 2-D bf16 tensor map with 64-column (128-byte) boxes and the 128-byte swizzle.
static bool map_bf16_sw128(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct ChunkLayoutSmem {
  int NC, NK, NRAW;
  bool rtc;
  uint32_t off_q, off_ar, off_p, off_c, off_k, off_raw, off_bar, off_misc, c_stage, k_stage, raw_stage, total;
};

// Shared memory: [Q_lat boxes][RoPE query boxes][P buffers][latent ring][RoPE-key ring]
// [code ring][barriers][misc].  With M = 64 the A operands' rows 32..63 read the 4 KB after
// each 32-row box (the next box, P0, or the first latent stage), all inside the allocation.
// The rings take what is left.  A key stage is free after MMA1 (RoPE scores on the tensor
// cores) or once the softmax warps hold its keys in registers, a latent stage only after
// MMA2, so the latent ring gets up to two stages more than the key ring.
static ChunkLayoutSmem chunk_smem_rtc(int dc, int R, int qbits, int rows, bool rtc) {
  const uint32_t budget = 232448 - 1024;
  const int dcp = (dc + 63) / 64 * 64;
  const int n_cbox = dcp / 64, n_kbox = (R + 63) / 64;
  ChunkLayoutSmem L{};
  L.rtc = rtc;
  L.c_stage = (uint32_t)n_cbox * kTBox;
  L.k_stage = (uint32_t)n_kbox * kTBox;
  L.raw_stage = qbits ? (((uint32_t)kCT * (dc * qbits / 8)) + 127) & ~127u : 0;
  L.NRAW = qbits ? 3 : 0;
  const uint32_t box = (uint32_t)rows * 128u;
  const uint32_t fixed = (uint32_t)(n_cbox + (rtc ? n_kbox : 0)) * box + 2 * box + L.NRAW * L.raw_stage;
  auto size = [&](int nc, int nk) {
    return fixed + nc * L.c_stage + nk * L.k_stage + 8 * (2 * nc + 2 * nk + 2 * L.NRAW + kFixedBars) + 16 + kXchgBytes + 256;
  };
  int nc = 2, nk = 2;
  while (true) {   // the latent ring up to two stages ahead of the key ring, then alternately
    const bool want_c = nc < nk + 2;
    if (want_c && nc < 6 && size(nc + 1, nk) <= budget) { ++nc; continue; }
    if (nk < nc && nk < 6 && size(nc, nk + 1) <= budget) { ++nk; continue; }
    if (nc < 6 && size(nc + 1, nk) <= budget) { ++nc; continue; }
    break;
  }
  L.NC = nc;
  L.NK = nk;
  uint32_t o = 0;
  L.off_q = o; o += (uint32_t)n_cbox * box;
  L.off_ar = o; o += rtc ? (uint32_t)n_kbox * box : 0;
  L.off_p = o; o += 2 * box;
  L.off_c = o; o += nc * L.c_stage;
  L.off_k = o; o += nk * L.k_stage;
  L.off_raw = o; o += L.NRAW * L.raw_stage;
  L.off_bar = o; o += 8 * (2 * nc + 2 * nk + 2 * L.NRAW + kFixedBars);
  o = (o + 15) & ~15u;
  L.off_misc = o; o += 16 + kXchgBytes;
  L.total = o + 1024;
  return L;
}

// The RoPE scores of a 128-row unit go to the tensor cores (block-diagonal query rows in
// MMA1) when their operand leaves room for at least three latent and two key stages; else,
// and always for 32 rows (whose MMA1 would double on mostly zero rows while only two
// softmax warps share the CUDA-core form), the softmax warps compute them from the key stage.
static ChunkLayoutSmem chunk_smem(int dc, int R, int qbits, int rows) {
  if (rows == 32) return chunk_smem_rtc(dc, R, qbits, rows, false);
  const ChunkLayoutSmem t = chunk_smem_rtc(dc, R, qbits, rows, true);
  if (t.total <= 232448 && t.NC >= 3 && t.NK >= 2) return t;
  return chunk_smem_rtc(dc, R, qbits, rows, false);
}

}  // namespace chunk
}  // namespace mla

// Shapes the kernel covers: bf16 with r = 4 kept pairs per KV head (2r = 8 RoPE dims, one
// 16-byte chunk per KV head), d_c a multiple of 32 up to 256 (the TMA boxes zero-fill a
// latent narrower than a multiple of 64), RoPE keys up to 256 dims, heads up to 128; the
// quantised caches with whole 16-byte code rows.
static bool attn_shape_ok(const mla_plan& p, int rows_cap) {
  const mla_config_t& cfg = p.cfg;
  if (cfg.dtype != MLA_BF16 || 2 * cfg.r_pairs != 8 || p.R > 256 || p.R % 8 != 0) return false;
  if (cfg.d_c % 32 != 0 || cfg.d_c > 256 || cfg.n_heads > 128) return false;
  const bool quant = mla_kind_quant(cfg.cache_kind);
  const int qbits = quant ? mla_quant_bits(cfg.cache_kind) : 0;
  if (quant && (cfg.d_c * qbits / 8) % 16 != 0) return false;
  return mla::chunk::chunk_smem(cfg.d_c, p.R, qbits, rows_cap).total <= 232448;
}

// Any cache view the validation accepts (the dequantising warps read scales with plain loads).
static bool attn_cache_ok(const mla_plan&, const mla_cache_t&) { return true; }

// Many queries per sequence: units of 128 / H queries x H heads (M = 128), without the
// residual window (it depends on each query's own length, so a tile's latent rows would
// differ between the queries that share it).
bool mla_chunk_capable(const mla_plan& p) {
  return p.cfg.cache_kind != MLA_CACHE_INT4_G32_R128 && attn_shape_ok(p, 128);
}

bool mla_chunk_supported(const mla_plan& p, const mla_cache_t& c) {
  return mla_chunk_capable(p) && attn_cache_ok(p, c);
}

// The decode form (one query per unit: M = 64 for up to 32 heads, else M = 128).
bool mla_decode_t_capable(const mla_plan& p) { return attn_shape_ok(p, p.cfg.n_heads <= 32 ? 32 : 128); }

bool mla_decode_t_supported(const mla_plan& p, const mla_cache_t& c) {
  return mla_decode_t_capable(p) && attn_cache_ok(p, c);
}

cudaError_t mla_launch_chunk_tc(const mla_plan& p, const mla_cache_t& c, const int32_t* seq_lens, int B, int Q,
                                const Sched& sched, const void* qlat, const float* qrope, float* opart,
                                float* mlpart, int P, int G, cudaStream_t s, int rows) {
  using namespace mla::chunk;
  const mla_config_t& cfg = p.cfg;
  const int dc = cfg.d_c, R = p.R, H = cfg.n_heads;
  const int qbits = mla_kind_quant(cfg.cache_kind) ? mla_quant_bits(cfg.cache_kind) : 0;
  const int qper = rows == 128 ? (Q > 1 ? 128 / H : 1) : 1;   // queries per unit
  const uint32_t code_row = (uint32_t)(dc * qbits / 8);
  const uint64_t crows = mla_cache_rows(c);
  CUtensorMap tm_c, tm_kr, tm_q;
  bool ok = map_bf16_sw128(&tm_kr, c.k_rope, R, crows, kCT) &&
            map_bf16_sw128(&tm_q, qlat, dc, (uint64_t)B * Q * H, (uint32_t)rows);
  if (qbits) {   // code rows, one 64-row box per tile, no swizzle
    EncodeTiledFn fn = encode_fn();
    cuuint64_t gdim[2] = {code_row, crows};
    cuuint64_t gstride[1] = {code_row};
    cuuint32_t box[2] = {code_row, (cuuint32_t)kCT};
    cuuint32_t es[2] = {1, 1};
    ok = ok && fn && fn(&tm_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, c.c_kv, gdim, gstride, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  } else {
    ok = ok && map_bf16_sw128(&tm_c, c.c_kv, dc, crows, kCT);
  }
  if (!ok) return cudaErrorInvalidValue;
  const ChunkLayoutSmem L = chunk_smem(dc, R, qbits, rows);
  ChunkArgs a;
  a.q_chunk = Q; a.nqb = (Q + qper - 1) / qper; a.d_c = dc; a.R = R; a.P = P; a.T_cap = c.T_cap;
  a.H = H; a.qper = qper; a.rows = qper * H; a.dcp = (dc + 63) / 64 * 64;
  a.scales = (const __half*)c.c_scales; a.code_row = code_row;
  a.sched = sched; a.seq_lens = seq_lens; a.qrope = qrope; a.opart = opart; a.mlpart = mlpart;
  a.cache = c; a.err = p.err;
  a.wait_ns = (uint64_t)p.opt_wait_us * 1000u;
  a.rtc = L.rtc ? 1 : 0;
  a.NC = L.NC; a.NK = L.NK; a.NRAW = L.NRAW;
  a.off_q = L.off_q; a.off_ar = L.off_ar; a.off_p = L.off_p; a.off_c = L.off_c; a.off_k = L.off_k;
  a.off_raw = L.off_raw; a.off_bar = L.off_bar; a.off_misc = L.off_misc;
  a.c_stage = L.c_stage; a.k_stage = L.k_stage; a.raw_stage = L.raw_stage;
  const bool paged = c.block_table != nullptr, resid = qbits == 4 && c.c_resid != nullptr;
  decltype(&attn_tc_kernel<128, 0, false, false>) kern;
  if (rows == 128)
    kern = qbits == 4 ? (paged ? attn_tc_kernel<128, 4, false, true> : attn_tc_kernel<128, 4, false, false>)
           : qbits == 2 ? (paged ? attn_tc_kernel<128, 2, false, true> : attn_tc_kernel<128, 2, false, false>)
                        : (paged ? attn_tc_kernel<128, 0, false, true> : attn_tc_kernel<128, 0, false, false>);
  else
    kern = qbits == 4 ? (resid ? (paged ? attn_tc_kernel<32, 4, true, true> : attn_tc_kernel<32, 4, true, false>)
                               : (paged ? attn_tc_kernel<32, 4, false, true> : attn_tc_kernel<32, 4, false, false>))
           : qbits == 2 ? (paged ? attn_tc_kernel<32, 2, false, true> : attn_tc_kernel<32, 2, false, false>)
                        : (paged ? attn_tc_kernel<32, 0, false, true> : attn_tc_kernel<32, 0, false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  if ((e = mla_profile_event(p, kProfAttention, false, s)) != cudaSuccess) return e;
  const int threads = rows == 32 && qbits ? Crew<32, 4>::WARPS * 32 : 256;
  e = mla_launch_kernel(kern, dim3(G), dim3(threads), L.total, s, p.opt_pdl, tm_c, tm_kr, tm_q, a);
  if (e != cudaSuccess) return e;
  return mla_profile_event(p, kProfAttention, true, s);
}
