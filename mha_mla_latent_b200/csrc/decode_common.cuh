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

// Single-block schedule builder.  Must be run by one whole CTA.
__device__ inline void build_schedule(const int32_t* __restrict__ seq_lens, int B, int T_cap,
                                      int tile, int G, Sched s, int32_t* err) {
  __shared__ int32_t s_carry[2];
  __shared__ int32_t s_tot;
  const int tid = threadIdx.x, nt = blockDim.x;
  // 1. tiles per sequence and exclusive prefix sums (tiles and non-empty count).
  if (tid == 0) { s_carry[0] = 0; s_carry[1] = 0; }
  __syncthreads();
  for (int base = 0; base < B; base += nt) {
    int b = base + tid;
    int nti = 0;
    if (b < B) {
      int L = seq_lens[b];
      if (L < 0 || L > T_cap) { raise_error(err, MLA_DEVERR_SEQ_LEN); L = 0; }
      nti = (L + tile - 1) / tile;
      s.seq_ntiles[b] = nti;
      s.seq_np[b] = 0;
      s.seq_first[b] = 0;
    }
    // serial scan by thread 0 over this chunk (B is small compared to the decode work)
    __syncthreads();
    if (tid == 0) {
      int c0 = s_carry[0], c1 = s_carry[1];
      for (int i = base; i < min(B, base + nt); ++i) {
        s.seq_tile0[i] = c0;
        s.seq_ne[i] = c1;
        c0 += s.seq_ntiles[i];
        c1 += s.seq_ntiles[i] > 0 ? 1 : 0;
      }
      s_carry[0] = c0; s_carry[1] = c1;
    }
    __syncthreads();
  }
  if (tid == 0) { s_tot = s_carry[0]; s.seq_ne[B] = s_carry[1]; }
  __syncthreads();
  const long long T = s_tot;

  // sequence containing global tile t (t < T): last b with seq_tile0[b] <= t
  auto seq_of = [&](long long t) {
    int lo = 0, hi = B;  // first b with tile0 > t, in [0, B]
    while (lo < hi) {
      int mid = (lo + hi) >> 1;
      if (s.seq_tile0[mid] > t) hi = mid; else lo = mid + 1;
    }
    return lo - 1;
  };
  // 2. pieces per worker, 3. serial exclusive scan into worker_first.
  for (int i = tid; i < G; i += nt) {
    long long c0 = (long long)i * T / G, c1 = (long long)(i + 1) * T / G;
    int np = 0;
    if (c0 < c1) {
      int b0 = seq_of(c0), b1 = seq_of(c1 - 1);
      np = s.seq_ne[b1 + 1] - s.seq_ne[b0];
    }
    s.worker_first[i + 1] = np;
  }
  __syncthreads();
  if (tid == 0) {
    s.worker_first[0] = 0;
    for (int i = 0; i < G; ++i) s.worker_first[i + 1] += s.worker_first[i];
  }
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
      int L = seq_lens[b];
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
  const int P = s.worker_first[G];
  for (int p = tid; p < P; p += nt) {
    int b = s.piece_b[p];
    if (p == 0 || s.piece_b[p - 1] != b) s.seq_first[b] = p;
    atomicAdd(&s.seq_np[b], 1);
  }
}

}  // namespace mla
