/*
 * mla_api.h — C ABI of the MHA2MLA latent-cache decode library (B200, sm_100a).
 *
 * The method (paper notes "MHA2MLA: Towards Economical Inference by Enabling
 * DeepSeek's Multi-Head Latent Attention in Any Transformer-based LLMs", ACL 2025,
 * §方法详解/整体框架 and §关键设计) converts an MHA layer in two steps: partial-RoPE
 * keeps, per head, the r frequency pairs with the largest 2-norm contribution, and
 * a joint SVD of the NoPE key and value projections gives one shared latent
 * c_kv = x W_dkv with per-head up-projections W_uk, W_uv.  Decoding then caches
 * only c_kv and the kept RoPE key dims.
 *
 * Conventions (all entry points):
 *   - Notation: d hidden, H query heads, n_kv KV heads (G = H/n_kv, head h uses KV
 *     head g = h / G), d_h head dim, r kept pairs per KV head, R = n_kv*2r,
 *     d_c latent width.  Pair k is the dims (2k, 2k+1); theta_k = base^(-2k/d_h);
 *     positions are 0-based.
 *   - Arrays are dense row-major (C order).  "dtype" means the config's dtype:
 *     MLA_F32 = IEEE float32, MLA_BF16 = bfloat16 (uint16 storage).
 *   - Pointers documented "device" must be device memory of the current device and
 *     16-byte aligned; "host" pointers are ordinary host memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is enqueued on it; calls return before it completes.
 *   - Every call validates its arguments first and returns a status without
 *     launching anything when they are bad.  MLA_ERR_CUDA reports a failed CUDA
 *     call (including an earlier asynchronous error surfacing at launch).
 *     Device-side conditions (a sequence length beyond the cache capacity, a
 *     pipeline wait that exceeded its bound) are recorded in the plan's device
 *     error word and read with mla_device_error().
 *   - The library never allocates device memory inside mla_append or mla_decode;
 *     the caller owns inputs, outputs, the cache and the workspace.  A plan owns
 *     its packed weight copies.  Calls on one plan are not thread-safe.
 */
#ifndef MLA_API_H
#define MLA_API_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,          /* null pointer, non-positive or inconsistent size */
  MLA_ERR_UNSUPPORTED = 2,          /* valid shape/dtype combination this build does not run */
  MLA_ERR_ALIGNMENT = 3,            /* a device pointer is not 16-byte aligned */
  MLA_ERR_WORKSPACE_TOO_SMALL = 4,  /* ws_bytes < mla_decode_workspace_bytes() */
  MLA_ERR_CUDA = 5,                 /* a CUDA runtime/driver call failed */
  MLA_ERR_DEVICE = 6                /* a kernel recorded an error (see mla_device_error) */
} mla_status_t;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype_t;

/* Latent cache encoding.  MLA_CACHE_SAME stores c_kv in the config dtype.
 * MLA_CACHE_INT4_G32 stores it per token in groups of 32 elements: one fp16
 * scale s = fp16(absmax/7) per group and 4-bit two's-complement codes
 * clamp(round_half_even(c/s), -7, 7) (codes 0 when s == 0), element 2i in the low
 * nibble of byte i; value = code*s.  (Notes §关键设计: 4-bit quantisation stacks on
 * the latent; the group layout is this library's choice.)  RoPE dims stay in dtype.
 * MLA_CACHE_INT4_G32_R128 is MLA_CACHE_INT4_G32 plus an unquantised residual window:
 * each sequence's MLA_RESID_WINDOW most recent tokens are read at full precision.  The
 * README "MHA2MLA" (§LongBench evaluation: the 4-bit HQQ quantised cache is run with a
 * residual length of 128) deploys the 4-bit cache this way.  Every token still gets its
 * int4 row; in addition the latent of token t, in dtype, goes to slot t % 128 of the
 * sequence's ring c_resid, and resid_pos[slot] records which position the slot holds
 * (the largest one appended there: it only grows).  Decode reads token t of a sequence
 * of length L from the ring when t >= L - 128 and resid_pos[t % 128] == t, else from the
 * int4 row, so with positions appended in order the window is exactly [L-128, L). */
typedef enum {
  MLA_CACHE_SAME = 0, MLA_CACHE_INT4_G32 = 1, MLA_CACHE_INT4_G32_R128 = 2, MLA_CACHE_INT2_G32 = 3
} mla_cache_kind_t;
/* MLA_CACHE_INT2_G32 is the same scheme at 2 bits (Notes §关键设计: 4-bit or 2-bit
 * quantisation stacks on the latent): per token, groups of 32, fp16 scale s = fp16(absmax),
 * codes clamp(round_half_even(c/s), -1, 1) (0 when s == 0), two's-complement 2-bit fields,
 * element 4i+k in bits 2k..2k+1 of byte i; value = code*s.  The quantised caches are
 * decoded on the tensor cores wherever the head-row kernel's shapes allow (dtype bf16,
 * r = 4, at most 128 query heads and 32 KV heads, d_c a multiple of 32 up to 256 whose
 * code rows are whole 16-byte chunks: a multiple of 64 at 2 bits) and on the CUDA cores
 * otherwise. */
#define MLA_RESID_WINDOW 128

typedef struct {
  int32_t hidden;       /* d */
  int32_t n_heads;      /* H, multiple of n_kv_heads */
  int32_t n_kv_heads;   /* n_kv */
  int32_t head_dim;     /* d_h, even */
  int32_t r_pairs;      /* r, 0 <= r <= d_h/2 */
  int32_t d_c;          /* latent width, multiple of 4 (of 32 for the int4 cache) */
  double rope_base;     /* RoPE base (10000 for the Llama/SmolLM shapes) */
  float softmax_scale;  /* score scale; 0 = 1/sqrt(d_h), the original layer's (must be >= 0) */
  int32_t dtype;        /* mla_dtype_t */
  int32_t cache_kind;   /* mla_cache_kind_t (the int4 and int2 kinds require dtype MLA_BF16) */
} mla_config_t;

/* Caller-owned cache, device memory, capacity T_cap tokens per sequence.
 * Contiguous (block_table == NULL): each sequence owns T_cap token rows, in the arrays below.
 * Paged (block_table != NULL): the arrays are pools of n_blocks blocks of MLA_BLOCK_TOKENS
 * (128) tokens, and token t of sequence b lives in token row t % 128 of pool block
 * block_table[b][t / 128]; every array below is then read with B := n_blocks and
 * T_cap := 128.  T_cap must be a
 * multiple of 128 (the logical capacity: T_cap / 128 table entries per sequence).  The
 * README "MHA2MLA" runs ragged LongBench batches; 128-token blocks match the decode tile,
 * so each tile of the attention kernel reads one block.  A table entry outside
 * [0, n_blocks) flags MLA_DEVERR_BLOCK and reads or writes block 0 instead.  The arrays
 * may hold at most 2^31 - 1 token rows (B * T_cap, or n_blocks * 128 when paged); a larger
 * view is refused with MLA_ERR_UNSUPPORTED.
 *   c_kv      SAME: [B][T_cap][d_c] dtype;  INT4*: [B][T_cap][d_c/2] uint8 codes;
 *             INT2: [B][T_cap][d_c/4] uint8 codes
 *   c_scales  INT4*, INT2: [B][T_cap][d_c/32] fp16;  SAME: must be NULL
 *   k_rope    [B][T_cap][n_kv][2r] dtype (may be NULL when r == 0): the kept RoPE key
 *             dims, one row of n_kv*2r values per token (token-major, like c_kv); element
 *             (b, t, g, j) sits at ((b*T_cap + t)*n_kv + g)*2r + j
 *   c_resid   INT4_G32_R128: [B][128][d_c] dtype, the residual ring; otherwise NULL
 *   resid_pos INT4_G32_R128: [B][128] int32, the position each ring slot holds; set every
 *             entry to -1 before a sequence's first append (and again when a sequence
 *             slot is reused for a new sequence); otherwise NULL */
typedef struct {
  void* c_kv;
  void* c_scales;
  void* k_rope;
  int32_t B;
  int32_t T_cap;
  void* c_resid;
  int32_t* resid_pos;
  const int32_t* block_table;   /* paged: device [B][T_cap/128] int32 pool block ids; else NULL */
  int32_t n_blocks;             /* paged: blocks in the pool; else 0 */
} mla_cache_t;
#define MLA_BLOCK_TOKENS 128

typedef struct mla_plan mla_plan_t;   /* opaque, created by mla_plan_create */

/* Options for mla_plan_set_option. */
enum {
  MLA_OPT_DECODE_KERNEL = 1,  /* 0 auto (see mla_decode_kernel_choice), 1 CUDA-core split-K
                                 kernel, 2 tcgen05 kernel with a token per softmax thread,
                                 3 tcgen05 kernel with a head per softmax thread (the
                                 query-chunk kernel's form, one query) */
  MLA_OPT_DECODE_SPLITS = 2,  /* 0 auto (SM count based); n > 0: split the context
                                 tiles into n contiguous worker ranges */
  MLA_OPT_PROFILE_EVENTS = 3, /* value: address of a host array of two cudaEvent_t; each
                                 mla_decode records [0] just before and [1] just after its
                                 split-K attention kernel on the call's stream (0 = off).
                                 The array must stay valid while the option is set. */
  MLA_OPT_OVERLAP_LAUNCH = 4, /* 1 (default): launch the kernels of mla_append / mla_decode
                                 with programmatic stream serialization, so each one's
                                 independent prologue (weight loads, set-up) overlaps the
                                 tail of the kernel before it; 0: plain stream order */
  MLA_OPT_WAIT_LIMIT_US = 5,  /* bound of every pipeline wait of the tensor-core decode
                                 kernel, in microseconds, 100 .. 10^7 (default 10^6 = 1 s).
                                 A wait that runs out sets MLA_DEVERR_TIMEOUT; the kernel
                                 then drains its copies, releases its tensor memory and
                                 returns, and the decode output of that call is invalid. */
  MLA_OPT_TEST_SKIP_COPY = 6, /* testing the timeout path only (0 = off, the default): with
                                 value k > 0 every CTA of the tensor-core kernel leaves out
                                 the latent copy of its k-th tile, so the waits for that tile
                                 run out (after MLA_OPT_WAIT_LIMIT_US) and the call reports
                                 MLA_DEVERR_TIMEOUT.  Nothing faults; later calls with the
                                 option cleared run normally. */
  MLA_OPT_PROFILE_KERNELS = 8  /* value: address of a host array of eight cudaEvent_t (0 =
                                 off); each call records [2k] just before and [2k+1] just
                                 after its kernel k on the call's stream: k = 0 the append
                                 kernel (mla_append), 1 the query absorption, 2 the split-K
                                 attention, 3 the split merge (mla_decode).  Events between
                                 kernels stop their launches from overlapping, so each
                                 interval times its kernel alone.  Overrides
                                 MLA_OPT_PROFILE_EVENTS while set. */
};

/* A static, NUL-terminated English name of a status ("unknown status" for a value outside
 * mla_status_t); never NULL, never to be freed. */
MLA_API const char* mla_status_string(mla_status_t s);
/* A static string naming this library build and its target (sm_100a); never NULL. */
MLA_API const char* mla_version(void);

/* Bytes cached per token per layer for this config (c_kv, scales, RoPE dims).
 * Notes §关键设计 (SVDjoint; KV-cache quantisation).  Returns 0 for an invalid config. */
MLA_API size_t mla_cache_bytes_per_token(const mla_config_t* cfg);

/* 2-norm contribution scores and head-wise top-r pair selection.
 * Notes §关键设计, contribution-aware partial-RoPE removal: the contribution of pair k
 * is bounded by ||q^[2k,2k+1]||*||k^[2k,2k+1]||; it is averaged over the T calibration
 * tokens and over the G query heads of each KV head, then the r largest pairs are kept
 * (equal scores: lower k first).  Accumulation is float32 in a fixed order.
 *   q_cal    device [T][H][d_h] dtype, unrotated calibration queries
 *   k_cal    device [T][n_kv][d_h] dtype, unrotated calibration keys
 *   pair_idx device out [n_kv][r] int32, ascending within each KV head
 *   contrib  device out [n_kv][d_h/2] float32 scores, or NULL               */
MLA_API mla_status_t mla_select_pairs(const mla_config_t* cfg, const void* q_cal, const void* k_cal,
                              int32_t T, int32_t* pair_idx, float* contrib, void* stream);

/* Fixed partial-RoPE strategies for mla_fixed_pairs. */
enum {
  MLA_PAIRS_HIGH = 1,
  MLA_PAIRS_UNIFORM = 2,
  MLA_PAIRS_LOW = 5,
  MLA_PAIRS_FULL = 0
};

/* Fixed partial-RoPE pair sets, the alternatives to the 2-norm selection that the README
 * "MHA2MLA" (§Fine-Tuning strategy tables: partial-RoPE versions) lists and the Notes
 * (§消融实验, Partial-RoPE strategy comparison) compare.  With P = d_h/2 pairs, r = r_pairs
 * and theta_k = base^(-2k/d_h) (k = 0 is the highest frequency):
 *   MLA_PAIRS_HIGH     k = 0 .. r-1            (highest frequencies)
 *   MLA_PAIRS_LOW      k = P-r .. P-1          (lowest frequencies)
 *   MLA_PAIRS_UNIFORM  k_j = floor(j*P/r), j = 0 .. r-1   (evenly spaced)
 *   MLA_PAIRS_FULL     every pair (requires r == P: full RoPE)
 * The same set is used for every KV head.  pair_idx: HOST [n_kv][r] int32, ascending.
 * Returns MLA_ERR_INVALID_ARG for an unknown strategy or r out of range.  No GPU use. */
MLA_API mla_status_t mla_fixed_pairs(const mla_config_t* cfg, int32_t strategy, int32_t* pair_idx);

/* Build a plan: validate the config and copy/pack the converted weights into
 * plan-owned device memory.  All weight pointers are HOST memory in the config dtype.
 *   W_dkv    [d][d_c]            joint-SVD down-projection (U_trunc)
 *   W_k      [d][n_kv*d_h]       original key projection; the plan keeps the columns
 *                                of the selected pairs (the RoPE key dims)
 *   pair_idx [n_kv][r] int32     selected pairs, ascending, each in [0, d_h/2)
 *   W_uk     [n_kv][d_c][d_h-2r] NoPE key up-projection (rows of Sigma V^T)
 *   W_uv     [n_kv][d_c][d_h]    value up-projection
 * Notes §关键设计 (SVDjoint): W_dkv = U_trunc, Sigma V^T split per head.
 * On success *out receives the plan; release it with mla_plan_destroy.  MLA_ERR_CUDA when
 * a device call fails or the host or device memory for the packed copies cannot be
 * allocated; *out is then NULL and nothing is left allocated. */
MLA_API mla_status_t mla_plan_create(const mla_config_t* cfg, const void* W_dkv, const void* W_k,
                             const int32_t* pair_idx, const void* W_uk, const void* W_uv,
                             mla_plan_t** out);
/* Release a plan and its device memory (cudaFree, which waits for the device to go idle).
 * NULL is a no-op.  No work that uses the plan may still be in flight on any stream. */
MLA_API void mla_plan_destroy(mla_plan_t* plan);
/* Set one MLA_OPT_* option (the enum above gives each option's values and meaning); it
 * applies to the calls made after it.  MLA_ERR_INVALID_ARG for a NULL plan, an unknown
 * option or a value outside the option's range; the plan is then unchanged. */
MLA_API mla_status_t mla_plan_set_option(mla_plan_t* plan, int32_t option, int64_t value);

/* Append N tokens to the cache.  For token n: c = x[n] W_dkv (float32 accumulation),
 * the RoPE key dims x[n] W_k[:, kept pairs of g] are rotated at position pos[n]
 * (angle computed in float64), c is stored in the cache encoding, and both are written
 * at (seq_idx[n], pos[n]).  Notes §关键设计 (SVDjoint: c_kv = x W_dkv; partial-RoPE).
 *   x       device [N][d] dtype
 *   seq_idx device [N] int32 in [0, B);  pos device [N] int32 in [0, T_cap)
 * Tokens with an out-of-range seq_idx/pos are skipped and flag the device error word.
 * Distinct tokens must target distinct (seq, pos) slots.  With the residual window
 * (MLA_CACHE_INT4_G32_R128) one call may carry any number of a sequence's tokens: a first
 * kernel raises resid_pos[slot] to the largest position of the call that maps to the slot,
 * and only that token writes the ring row. */
MLA_API mla_status_t mla_append(const mla_plan_t* plan, const void* x, const int32_t* seq_idx,
                        const int32_t* pos, int32_t N, const mla_cache_t* cache, void* stream);

/* Device workspace mla_decode, mla_decode_step and mla_decode_step_host need for a batch
 * of B sequences (bytes, 256-aligned; it includes the host variant's staging of the step's
 * inputs and output).  0 for a NULL plan or B <= 0. */
MLA_API size_t mla_decode_workspace_bytes(const mla_plan_t* plan, int32_t B);

/* The attention kernel mla_decode runs for this plan and cache under the plan's
 * MLA_OPT_DECODE_KERNEL setting: *kernel = 1 (CUDA cores), 2 (tcgen05, a token per softmax
 * thread) or 3 (tcgen05, a head per softmax thread), the option's own numbering.  Automatic
 * choice (option 0): kernel 3 where its shapes allow, else kernel 2, else kernel 1.  Host
 * only; no device work.  Returns MLA_ERR_UNSUPPORTED where the forced kernel cannot run the
 * shape, MLA_ERR_INVALID_ARG for null arguments. */
MLA_API mla_status_t mla_decode_kernel_choice(const mla_plan_t* plan, const mla_cache_t* cache, int32_t* kernel);

/* One decode step: attention of each sequence's new query over its cached tokens
 * [0, seq_lens[b]).  The query sits at position seq_lens[b]-1 (append it first).
 * Steps: split q into NoPE and kept-RoPE dims; rotate the RoPE part; absorb W_uk into
 * the NoPE part (q_lat = q_nope W_uk^T) so it scores against c_kv directly; add the
 * RoPE score; scale 1/sqrt(d_h); split-K online softmax over the context; accumulate
 * the probability-weighted latent; merge the splits; apply W_uv per head.
 * Notes §关键设计 (the RoPE part cannot join the matrix merge and is computed apart).
 *   seq_lens device [B] int32 (0 <= L <= T_cap; L == 0 gives a zero output row)
 *   q        device [B][H][d_h] dtype, unrotated, original dim order
 *   out      device [B][H][d_h] dtype, per-head attention output (before W_o)
 *   workspace device, >= mla_decode_workspace_bytes(plan, B) bytes              */
MLA_API mla_status_t mla_decode(const mla_plan_t* plan, const mla_cache_t* cache, const int32_t* seq_lens,
                        const void* q, int32_t B, void* out, void* workspace, size_t ws_bytes,
                        void* stream);

/* Device workspace of mla_decode_chunk for B sequences of Q queries (bytes, 256-aligned;
 * 0 for a NULL plan or B, Q <= 0). */
MLA_API size_t mla_decode_chunk_workspace_bytes(const mla_plan_t* plan, int32_t B, int32_t Q);

/* Many queries per sequence, causally: the newest Q tokens of each sequence (a chunk of a
 * long document being prefilled, or drafted tokens to verify) attend over the cache in one
 * call.  seq_lens[b] counts all of sequence b's cached tokens, the chunk's own included
 * (append them first); query i (0 <= i < Q) of sequence b sits at position
 * p = seq_lens[b] - Q + i, is rotated there, and attends over tokens [0, p].  Per query this
 * is exactly mla_decode with length p + 1.  The queries of a sequence share the cache tiles
 * they read: blocks of floor(128/H) queries x H heads (at most 128 score rows) are scored
 * against each tile together on the tensor cores, so a block streams its prefix once.  Notes §方法详解/整体框架 and §关键设计 (absorbed latent scores plus the
 * separate RoPE term); the README "MHA2MLA" evaluates long documents (LongBench).
 *   seq_lens  device [B] int32, Q <= L <= T_cap
 *   q         device [B][Q][H][d_h] dtype, unrotated, original dim order
 *   out       device [B][Q][H][d_h] dtype, per-head attention output (before W_o)
 *   workspace device, >= mla_decode_chunk_workspace_bytes(plan, B, Q) bytes
 * Q == 1 is mla_decode.  For Q > 1 this build needs the head-row kernel's shapes (dtype
 * bf16, r = 4, at most 128 query heads and 32 KV heads, d_c a multiple of 32 up to 256;
 * bf16, int4 or int2 latent cache, paged or contiguous) and no residual window
 * (MLA_CACHE_INT4_G32_R128: each query's window depends on its own position).  Otherwise,
 * and with MLA_OPT_DECODE_KERNEL = 1, it returns MLA_ERR_UNSUPPORTED; one mla_decode per
 * query through per-query views of a paged cache covers those shapes. */
MLA_API mla_status_t mla_decode_chunk(const mla_plan_t* plan, const mla_cache_t* cache, const int32_t* seq_lens,
                                      const void* q, int32_t B, int32_t Q, void* out, void* workspace,
                                      size_t ws_bytes, void* stream);

/* One serving-loop decode step in a single call: the append of every sequence's new
 * token, then the decode of every sequence's new query.  Token b (row b of x) is the
 * newest token of sequence b: it is appended at position seq_lens[b] - 1 (the length
 * already counts it), and query b then attends over tokens [0, seq_lens[b]).  The result
 * equals mla_append(x, seq_idx = 0..B-1, pos = seq_lens - 1) followed by mla_decode;
 * the append and the query absorption, which do not depend on each other, run in one
 * launch (bf16, B <= 128), so a step is three kernels.  Notes §关键设计 (the cache holds
 * c_kv = x W_dkv and the kept RoPE key dims; decode absorbs W_uk and applies W_uv after
 * the weighted sum).  With the residual window, each new token claims its ring slot itself.
 *   seq_lens  device [B] int32, 1 <= L <= T_cap
 *   x         device [B][d] dtype, the new tokens' hidden states
 *   q         device [B][H][d_h] dtype, unrotated queries
 *   out       device [B][H][d_h] dtype
 *   workspace device, >= mla_decode_workspace_bytes(plan, B) bytes              */
MLA_API mla_status_t mla_decode_step(const mla_plan_t* plan, const mla_cache_t* cache, const int32_t* seq_lens,
                                     const void* x, const void* q, int32_t B, void* out, void* workspace,
                                     size_t ws_bytes, void* stream);

/* mla_decode_step with the step's inputs and output in HOST memory (page-locked memory
 * lets the copies run asynchronously): seq_lens [B] int32, x [B][d], q [B][H][d_h] and out
 * [B][H][d_h] are host pointers; the cache and the workspace are device memory.  The call
 * enqueues the host-to-device copies of seq_lens, x and q into the workspace, the step's
 * kernels, and the device-to-host copy of the output, all on `stream`: out is complete
 * once the stream reaches that point (e.g. after cudaStreamSynchronize).  The host buffers
 * must stay untouched until then.  workspace >= mla_decode_workspace_bytes(plan, B). */
MLA_API mla_status_t mla_decode_step_host(const mla_plan_t* plan, const mla_cache_t* cache, const int32_t* seq_lens,
                                          const void* x, const void* q, int32_t B, void* out, void* workspace,
                                          size_t ws_bytes, void* stream);

/* Size of the static scratch array behind mla_decode_noalloc (bytes, per device). */
#define MLA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* mla_decode without any device allocation, by the caller or by the library.
 * The paper has no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory when they decode: a server whose memory pool is carved up
 * once at start-up, a real-time loop that must not call the allocator (an allocation
 * can synchronise the device and has no bounded latency), or a host program that only
 * links this C ABI and has no allocator of its own.  Arguments, outputs and results are
 * those of mla_decode, minus the workspace: the workspace is a static device array of
 * MLA_NOALLOC_SCRATCH_BYTES compiled into the library, present on every GPU that loads
 * the library until the process exits.
 *   - Returns MLA_ERR_WORKSPACE_TOO_SMALL when the batch needs more workspace than the
 *     array holds (mla_decode_workspace_bytes(plan, B) tells how much a batch needs).
 *   - The first successful call on a device looks up the array's device address (with
 *     that device current) and keeps it; a failed lookup returns MLA_ERR_CUDA, leaves no
 *     pending CUDA error behind and is retried by the next call.  Make the first call
 *     before any stream capture.
 *   - The plan must belong to the current device (MLA_ERR_INVALID_ARG otherwise).
 *   - All calls share the one array and each leaves its contents behind.  Nothing in
 *     it needs clearing: every call writes each part of the workspace before reading it.
 *     Calls whose work overlaps on the GPU (different streams, or different plans on
 *     concurrent streams) race on the array; serialise them, e.g. on one stream.
 *   - It calls no cudaMalloc/cudaFree or other allocating routine. */
MLA_API mla_status_t mla_decode_noalloc(const mla_plan_t* plan, const mla_cache_t* cache,
                                        const int32_t* seq_lens, const void* q, int32_t B, void* out,
                                        void* stream);

/* Device error bits (the plan's device error word). */
enum {
  MLA_DEVERR_SEQ_LEN = 1,     /* a seq_lens entry was < 0 or > T_cap (treated as 0) */
  MLA_DEVERR_APPEND_SLOT = 2, /* an append token had seq_idx/pos out of range (skipped) */
  MLA_DEVERR_TIMEOUT = 4,     /* a pipeline wait exceeded its bound (output invalid) */
  MLA_DEVERR_BLOCK = 8        /* a paged cache's block table named a block outside the pool */
};
/* Synchronise the device, read and clear the plan's device error word.
 * *code receives 0 (none) or a bitwise OR of MLA_DEVERR_* values.
 * Returns MLA_OK, MLA_ERR_INVALID_ARG for a NULL plan or code, or MLA_ERR_CUDA when the
 * synchronisation itself failed. */
MLA_API mla_status_t mla_device_error(mla_plan_t* plan, int32_t* code);

#ifdef __cplusplus
}
#endif

#endif /* MLA_API_H */
