// Split-K schedule shared by the decode kernels and the combine.
//
// The context of every sequence is cut into tiles of `tile` tokens; the tiles of all
// sequences, laid end to end, are divided into G contiguous worker ranges of nearly
// equal size (worker i takes global tiles [floor(i*T/G), floor((i+1)*T/G))).  A
// "piece" is the part of one sequence inside one worker range; each piece yields one
// partial (running max m, sum l, unnormalised latent O) that the combine merges.
// Balanced ranges keep every SM busy whatever the length mix (ragged batches).
#pragma once

#include "common.cuh"

namespace mla {

// Block-wide exclusive scan of one int per thread (blockDim.x a multiple of 32, <= 1024).
// Returns the exclusive prefix; *total receives the block sum.  Uses s_warp[32].
__device__ inline int block_exscan(int v, int* total, int* s_warp) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int wv = lane < nw ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, wv, o);
      if (lane >= o) wv += y;
    }
    s_warp[lane] = wv;  // inclusive warp totals
  }
  __syncthreads();
  const int base = wid > 0 ? s_warp[wid - 1] : 0;
  *total = s_warp[nw - 1];
  __syncthreads();
  return base + x - v;
}

// Single-block schedule builder.  Must be run by one whole CTA.  It first waits for the
// kernel before (the sequence lengths are the caller's input and the workspace may still
// be read by the previous call).  When `scratch` (shared memory, `scratch_ints` ints) can
// hold all of it, the schedule is built there and copied out once, coalesced; otherwise
// it is built in the workspace directly.
// Many queries per sequence (q_chunk > 1): the schedule runs over units v = (sequence b =
// v / nqb, block k = v % nqb of q_block consecutive queries) and unit v's length is the
// last position of its block + 1: L_b - q_chunk + min(q_chunk, (k + 1) q_block) tokens,
// L_b = seq_lens[b] counting the chunk's own tokens.  B is then the number of units.
__device__ __forceinline__ int unit_len(const int32_t* __restrict__ seq_lens, int v, int q_chunk, int q_block) {
  if (q_chunk <= 1) return __ldg(seq_lens + v);
  const int nqb = (q_chunk + q_block - 1) / q_block, k = v % nqb;
  const int L = __ldg(seq_lens + v / nqb);
  return L < q_chunk ? -1 : L - q_chunk + min(q_chunk, (k + 1) * q_block);
}

__device__ inline void build_schedule(const int32_t* __restrict__ seq_lens, int B, int T_cap,
                                      int tile, int G, Sched out, int32_t* err, int32_t* scratch,
                                      int scratch_ints, int q_chunk = 1, int q_block = 1) {
  __shared__ int s_warp[32];
  const int tid = threadIdx.x, nt = blockDim.x;
  const int Pcap = B + G;
  const bool local = scratch && (long long)9 * B + 4 * G + 2 <= scratch_ints;
  Sched s = out;
  int32_t* seq_len = nullptr;
  pdl_wait();
  pdl_trigger();
  if (local) {
    int32_t* q = scratch;
    s.seq_tile0 = q; q += B;
    s.seq_ntiles = q; q += B;
    s.seq_ne = q; q += B + 1;
    s.seq_first = q; q += B;
    s.seq_np = q; q += B;
    s.worker_first = q; q += G + 1;
    s.piece_b = q; q += Pcap;
    s.piece_t0 = q; q += Pcap;
    s.piece_t1 = q; q += Pcap;
    seq_len = q;  // [B]
  }
  // 1. tiles per sequence; exclusive prefix sums of tiles and of non-empty sequences
  int carry_t = 0, carry_ne = 0;
  for (int base = 0; base < B; base += nt) {
    const int b = base + tid;
    int nti = 0;
    if (b < B) {
      int L = unit_len(seq_lens, b, q_chunk, q_block);
      if (L < 0 || L > T_cap) { raise_error(err, MLA_DEVERR_SEQ_LEN); L = 0; }
      nti = (L + tile - 1) / tile;
      s.seq_ntiles[b] = nti;
      if (seq_len) seq_len[b] = L;
      s.seq_np[b] = 0;
      s.seq_first[b] = 0;
    }
    int tot_t, tot_ne;
    const int ex_t = block_exscan(nti, &tot_t, s_warp);
    const int ex_ne = block_exscan(nti > 0 ? 1 : 0, &tot_ne, s_warp);
    if (b < B) {
      s.seq_tile0[b] = carry_t + ex_t;
      s.seq_ne[b] = carry_ne + ex_ne;
    }
    carry_t += tot_t;
    carry_ne += tot_ne;
  }
  if (tid == 0) s.seq_ne[B] = carry_ne;
  __syncthreads();
  const long long T = carry_t;

  // sequence containing global tile t (t < T): last b with seq_tile0[b] <= t; it is
  // non-empty because empty sequences share their start with the next sequence
  auto seq_of = [&](long long t) {
    int lo = 0, hi = B;
    while (lo < hi) {
      int mid = (lo + hi) >> 1;
      if (s.seq_tile0[mid] > t) hi = mid; else lo = mid + 1;
    }
    return lo - 1;
  };
  // 2./3. pieces per worker and their exclusive prefix (worker_first)
  int carry_p = 0;
  for (int base = 0; base < G; base += nt) {
    const int i = base + tid;
    int np = 0;
    if (i < G) {
      long long c0 = (long long)i * T / G, c1 = (long long)(i + 1) * T / G;
      if (c0 < c1) {
        int b0 = seq_of(c0), b1 = seq_of(c1 - 1);
        np = s.seq_ne[b1 + 1] - s.seq_ne[b0];
      }
    }
    int tot;
    const int ex = block_exscan(np, &tot, s_warp);
    if (i < G) s.worker_first[i] = carry_p + ex;
    carry_p += tot;
  }
  if (tid == 0) s.worker_first[G] = carry_p;
  __syncthreads();
  // 4. write pieces
  for (int i = tid; i < G; i += nt) {
    long long c0 = (long long)i * T / G, c1 = (long long)(i + 1) * T / G;
    if (c0 >= c1) continue;
    int pidx = s.worker_first[i];
    long long t = c0;
    int b = seq_of(t);
    while (t < c1) {
      long long e = (long long)s.seq_tile0[b] + s.seq_ntiles[b];
      if (e > c1) e = c1;
      int L = seq_len ? seq_len[b] : unit_len(seq_lens, b, q_chunk, q_block);
      if (L < 0 || L > T_cap) L = 0;
      s.piece_b[pidx] = b;
      s.piece_t0[pidx] = (int)((t - s.seq_tile0[b]) * tile);
      s.piece_t1[pidx] = (int)min((long long)L, (e - s.seq_tile0[b]) * tile);
      ++pidx;
      t = e;
      ++b;
      while (t < c1 && b < B && s.seq_ntiles[b] == 0) ++b;
    }
  }
  __syncthreads();
  // 5. per-sequence piece ranges (pieces are ordered by global tile, hence by sequence)
  const int P = carry_p;
  for (int p = tid; p < P; p += nt) {
    int b = s.piece_b[p];
    if (p == 0 || s.piece_b[p - 1] != b) s.seq_first[b] = p;
    atomicAdd(&s.seq_np[b], 1);
  }
  if (local) {   // copy the schedule out (coalesced)
    __syncthreads();
    for (int i = tid; i < B; i += nt) {
      out.seq_tile0[i] = s.seq_tile0[i];
      out.seq_ntiles[i] = s.seq_ntiles[i];
      out.seq_first[i] = s.seq_first[i];
      out.seq_np[i] = s.seq_np[i];
    }
    for (int i = tid; i <= B; i += nt) out.seq_ne[i] = s.seq_ne[i];
    for (int i = tid; i <= G; i += nt) out.worker_first[i] = s.worker_first[i];
    for (int i = tid; i < P; i += nt) {
      out.piece_b[i] = s.piece_b[i];
      out.piece_t0[i] = s.piece_t0[i];
      out.piece_t1[i] = s.piece_t1[i];
    }
  }
}

}  // namespace mla
