/*
 * starkv.h — C ABI of the STAR-KV latent decode-attention library (sm_100a).
 *
 * STAR-KV ("Low-Rank KV Cache Compression via Soft Thresholding for Adaptive
 * Rank Control", arXiv 2606.08382) keeps, per token and layer, low-dimensional
 * latents instead of full keys and values:
 *   - keys, head-wise:  Z_k,h = X A_k,h  (rank r_h per KV head), K_h = Z_k,h B_k,h
 *   - values, jointly:  Z_v   = X A_v    (rank r_v per layer),  V = Z_v B_v
 * (reading notes "STAR-KV 阅读笔记", sections 2.2, 5.1-5.2).  Keys are cached
 * before RoPE and reconstructed, rotated and scored on chip; the value
 * up-projection is folded into the output projection, M_h = B_v,h W_o,h, and
 * applied after aggregation (section 5.3).  Latents may carry a block-wise
 * Hadamard rotation absorbed into the factors and a 4/3-bit mixed-precision
 * quantization by singular-value order (section 6.1).  The decode data flow
 * is the notes' Algorithm 2.
 *
 * Conventions for every call below
 *   - Pointers named *host* are host memory; every other buffer pointer is
 *     device memory on the current CUDA device.  The caller owns all of them.
 *   - Row-major layouts; sizes are element counts unless stated in bytes.
 *   - Alignment: the pool, q, out, input and workspace buffers of the
 *     append, decode and prefill calls start on a 16-byte boundary, their
 *     int32 arrays on a 4-byte one (cudaMalloc and framework allocators give
 *     both).  A misaligned pointer returns STARKV_ERR_ARG before any launch.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never allocate device memory, except
 *     starkv_load_factors, which allocates the layer's own folded factors.
 *   - Errors found on the host return at once, before any launch, with a
 *     message available from starkv_last_error().  Errors found by a kernel
 *     (a page id outside the pool, a position outside the page table, a
 *     sequence length above the page table's capacity, an fp16 scale
 *     overflow, a bounded wait that expired) set the layer's device status
 *     word; no kernel traps.  starkv_sync_status() reads and clears it.
 *   - Not thread-safe per layer: calls on one layer from several host threads
 *     must be serialised by the caller.
 */
#ifndef STARKV_H
#define STARKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define STARKV_API __attribute__((visibility("default")))
#else
#define STARKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* starkv_stream_t;   /* same type as cudaStream_t */

typedef enum {
  STARKV_OK = 0,
  STARKV_ERR_ARG = 1,          /* invalid argument (null pointer, bad size, bad shape) */
  STARKV_ERR_UNSUPPORTED = 2,  /* valid, but not a combination the library implements */
  STARKV_ERR_OOM = 3,          /* device allocation failed (load only) */
  STARKV_ERR_CUDA = 4,         /* a CUDA runtime call failed */
  STARKV_ERR_DEVICE = 5,       /* the device status word was set (see starkv_sync_status) */
  STARKV_ERR_TIMEOUT = 6,      /* a bounded device-side wait expired */
  STARKV_ERR_WORKSPACE = 7     /* workspace smaller than starkv_workspace_bytes() */
} starkv_status;

/* Bits of the device status word. */
#define STARKV_DEV_BAD_PAGE      0x1   /* page_table entry outside [0, n_pages) */
#define STARKV_DEV_BAD_POSITION  0x2   /* append position outside the page table */
#define STARKV_DEV_SCALE_OVF     0x4   /* amax/qmax above the largest fp16 (65504) */
#define STARKV_DEV_TIMEOUT       0x8   /* a bounded wait gave up */

typedef enum { STARKV_F32 = 0, STARKV_BF16 = 1 } starkv_dtype;

/*
 * One attention layer.
 *   hidden D, n_heads H, n_kv_heads H_kv (H % H_kv == 0; query head h uses KV
 *   head h / (H / H_kv)), head_dim d (even, <= 256).
 *   key_ranks: host array [H_kv], each 1..d (ignored when plain).
 *   value_rank r_v: 1..H_kv*d (ignored when plain).
 *   dtype: element type of the factors, q, out and of unquantized latents.
 *   quantized: 0 = latents stored in dtype; 1 = 4/3-bit codes with an fp16
 *     scale per (token, group).  Channels [0, ceil(top_fraction*r)) use
 *     top_bits, the rest bottom_bits ("STAR-KV 阅读笔记" section 6.1;
 *     top_fraction 0.25, 4 and 3 bits on the model card
 *     "tenosra/longchat-7b-starkv-proxima").  Bits must be 2..8.
 *   group_size: channels per scale group, cut from the start of each segment;
 *     1..32.
 *   hadamard_block: 0 = no rotation; otherwise must equal group_size and
 *     requires quantized = 1.  Each group is rotated by a direct sum of
 *     normalised Sylvester-Hadamard blocks over the binary decomposition of its
 *     length (section 6.1: rotate the high-magnitude block and the ordinary
 *     block separately; absorbed into the factors).
 *   rope: 1 = rotate-half RoPE with base rope_theta on keys (at their slot
 *     position) and on the query (at q_pos).
 *   softmax_scale: 0 selects 1/sqrt(d).
 *   page_size: tokens per page; must be 16.
 *   plain: 1 = uncompressed layer (protected layers 0, 1 and 31 in the notes'
 *     Algorithm 1): K (after RoPE) and V are stored in dtype, width d per
 *     KV head each; no factors.
 *   max_positions: length of the layer's RoPE table for the tensor-core score
 *     kernel (0 selects 32768); 256 bytes of device memory per position.
 *     Decodes whose page table reaches beyond it use the CUDA-core path.
 *   unfused_output: 0 (default) = value-side output fusion, out = sum_h y_h M_h
 *     with M_h = B_v,h W_o,h folded at load (section 5.3); 1 = the same
 *     product in the other order, z_h = y_h B_v,kv(h) then out = z W_o,
 *     which reads H d (r_v + D) factor values per step instead of
 *     H r_v D (section 5.3 states the fusion as an exact reorder).  Needs a
 *     bf16 compressed layer with head_dim 128 and value_rank a multiple of 64.
 */
typedef struct {
  int hidden, n_heads, n_kv_heads, head_dim;
  const int* key_ranks;
  int value_rank;
  int dtype;
  int quantized;
  float top_fraction;
  int top_bits, bottom_bits;
  int group_size;
  int hadamard_block;
  int rope;
  double rope_theta;
  float softmax_scale;
  int page_size;
  int plain;
  int max_positions;
  int unfused_output;
} starkv_layer_config;

typedef struct starkv_layer starkv_layer;   /* opaque */

/* Sizes of one layer's stored state. */
typedef struct {
  int n_latents;            /* H_kv key latents + 1 value latent (plain: H_kv K + 1 V of width H_kv*d) */
  int latent_total;         /* sum of latent widths: R_k + r_v (plain: 2*H_kv*d) */
  int key_rank_total;       /* R_k = sum of key ranks (plain: H_kv*d) */
  size_t page_bytes;        /* bytes of one 16-token page, a multiple of 128 */
  double bytes_per_token;   /* algorithmic cache bytes per token (codes + scales, no padding) */
  size_t factor_bytes;      /* bytes decode reads from the layer's factors per step (B_k' + M, or B_k' + B_v + W_o unfused) */
} starkv_layer_info;

/*
 * Fold and upload the factors of one layer (Algorithm 1 steps 8-9 of the
 * notes, deploy side; section 5.3 for M_h; section 6.1 for the rotation).
 * Inputs are device pointers in cfg->dtype, unrotated:
 *   A_k [H_kv] blocks of D x r_h, concatenated in head order  (plain: W_k, D x H_kv*d)
 *   B_k [H_kv] blocks of r_h x d, concatenated                 (plain: NULL)
 *   A_v D x r_v                                                (plain: W_v, D x H_kv*d)
 *   B_v r_v x (H_kv*d)                                         (plain: NULL)
 *   W_o (H*d) x D
 * The layer keeps its own copies: A_k|A_v for the append projection, the
 * rotated key up-projections B'_k = R^T B_k, and M_h = B'_v,kv(h) W_o,h for
 * every query head, in the layout the kernels read.  The inputs may be freed
 * after the call returns and `stream` has been synchronised.
 * On success *out receives the layer; free it with starkv_free_layer.
 */
STARKV_API starkv_status starkv_load_factors(const starkv_layer_config* cfg, const void* A_k, const void* B_k,
                                  const void* A_v, const void* B_v, const void* W_o, starkv_stream_t stream,
                                  starkv_layer** out);

STARKV_API void starkv_free_layer(starkv_layer* layer);

STARKV_API starkv_status starkv_layer_get_info(const starkv_layer* layer, starkv_layer_info* info);

/* Bytes of one page of this layer. */
STARKV_API size_t starkv_page_bytes(const starkv_layer* layer);

/*
 * Zero n_pages pages of the pool (pool must be 16-byte aligned).  Appends OR
 * codes into zeroed pages, so a page must be zeroed before its first slot is
 * written, and again before it is reused for another sequence.
 */
STARKV_API starkv_status starkv_cache_init(const starkv_layer* layer, void* pool, int64_t n_pages, starkv_stream_t stream);

/*
 * Append n_tokens new tokens to the paged latent cache (Algorithm 2 steps 1-3).
 *   pool: n_pages pages of starkv_page_bytes() each, 16-byte aligned.
 *   page_table: int32 [n_seqs][max_pages]; token t of sequence b lives in
 *     page page_table[b][t / 16], slot t % 16.
 *   seq_idx: int32 [n_tokens], the sequence (row of page_table, < n_seqs) of each token.
 *   positions: int32 [n_tokens], the token's position in its sequence.
 *   input: input_is_latent = 0: hidden states x, [n_tokens][D] in dtype; the
 *            kernel projects z = x [A_k | A_v], applies the block rotation,
 *            quantizes and packs (plain layers: K = RoPE(x W_k), V = x W_v).
 *          input_is_latent = 1: float32 latents after rotation,
 *            [n_tokens][latent_total], in latent order (plain: K after RoPE,
 *            then V); the kernel only quantizes (or rounds) and packs.
 *   workspace: at least starkv_append_workspace_bytes(layer, n_tokens) bytes
 *     (may be NULL when that is 0).
 * Tokens of one call must go to distinct (sequence, position) slots whose
 * bytes are still zero.  This is the caller's obligation: the kernel checks
 * only that a position lies inside the page table (else
 * STARKV_DEV_BAD_POSITION) and that its page id lies inside the pool (else
 * STARKV_DEV_BAD_PAGE).  Codes are ORed into the slot, so writing a slot that
 * already holds a token corrupts it.  Packed bytes are bit-exact for given
 * float32 latents.  max_pages * 16 must fit in an int (else STARKV_ERR_ARG).
 */
STARKV_API starkv_status starkv_append(const starkv_layer* layer, void* pool, int64_t n_pages, const int32_t* page_table,
                            int n_seqs, int max_pages, int n_tokens, const int32_t* seq_idx, const int32_t* positions,
                            const void* input, int input_is_latent, void* workspace, size_t ws_bytes,
                            starkv_stream_t stream);

STARKV_API size_t starkv_append_workspace_bytes(const starkv_layer* layer, int n_tokens);

/*
 * Decode attention for one new query per sequence (Algorithm 2 steps 4-8).
 *   seq_lens: int32 [batch]; sequence b attends to slots [0, seq_lens[b]).
 *     A length of 0 gives a zero output row; a length above max_pages * 16
 *     sets STARKV_DEV_BAD_POSITION and is clamped.  max_pages * 16 must fit
 *     in an int (else STARKV_ERR_ARG).
 *   q_pos: int32 [batch] RoPE position of each query, or NULL for seq_lens[b]-1.
 *   q: [batch][H][d] in dtype (before RoPE).   out: [batch][D] in dtype.
 *   workspace: at least starkv_workspace_bytes(layer, batch, max_pages * 16, 1)
 *     bytes (the page table's capacity sets the score buffer's row length).
 */
STARKV_API starkv_status starkv_decode_attn(const starkv_layer* layer, const void* pool, int64_t n_pages,
                                 const int32_t* page_table, int max_pages, int batch, const int32_t* seq_lens,
                                 const int32_t* q_pos, const void* q, void* out, void* workspace, size_t ws_bytes,
                                 starkv_stream_t stream);

/*
 * Causal prefill attention over the cache (the tokens must already be
 * appended).  Sequence b has q_len[b] queries at positions q_start[b] ..
 * q_start[b] + q_len[b] - 1; query i attends to slots [0, q_start[b] + i].
 *   q_start_host, q_len_host: HOST int32 arrays [batch] (they set the launch shape).
 *   q: [sum q_len][H][d] in dtype, sequences one after another; out: [sum q_len][D].
 *   workspace: at least starkv_workspace_bytes(layer, batch, max_ctx, max q_len)
 *     bytes, where max_ctx >= every q_start[b] + q_len[b].
 * Paths, in order of preference:
 *   - bf16 layers with head_dim 128 (plain layers; compressed layers that the
 *     tensor-core decode takes, with key ranks <= 64 and positions inside
 *     the RoPE table): per sequence the chunk's keys and values are rebuilt
 *     once (K = RoPE(Zhat_k B'_k), V = Zhat_v B'_v, section 5.3 of the
 *     reading notes), then tiled causal attention and the output through W_o,
 *     all on the tensor cores.  Asynchronous on `stream`.
 *   - other tensor-core layers: every query row as a decode row, 256 rows at a
 *     time, when max_ctx is the page table's capacity (max_pages * 16).
 *   - the CUDA-core kernels otherwise.
 *   The last two copy a per-row table from pageable host memory and
 *   synchronise `stream` before returning.
 */
STARKV_API starkv_status starkv_prefill_attn(const starkv_layer* layer, const void* pool, int64_t n_pages,
                                  const int32_t* page_table, int max_pages, int batch, const int32_t* q_start_host,
                                  const int32_t* q_len_host, const void* q, void* out, void* workspace,
                                  size_t ws_bytes, starkv_stream_t stream);

/*
 * Workspace bytes for a decode of `batch` sequences (max_q = 1) or a prefill
 * of `batch` sequences with up to max_q queries each, over a page table whose
 * capacity is max_ctx tokens (max_pages * 16).  0 for a NULL layer.  The size
 * covers whichever kernel path the layer can take (tensor-core or CUDA-core).
 */
STARKV_API size_t starkv_workspace_bytes(const starkv_layer* layer, int batch, int max_ctx, int max_q);

/*
 * Synchronise `stream`, then read and clear the layer's device status word.
 * Returns STARKV_OK if it was zero, else STARKV_ERR_DEVICE (or
 * STARKV_ERR_TIMEOUT when only the timeout bit was set); *bits (may be NULL)
 * receives the word.
 */
STARKV_API starkv_status starkv_sync_status(const starkv_layer* layer, starkv_stream_t stream, uint32_t* bits);

/*
 * Decode attention without a caller-provided workspace.  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory themselves — for example a plugin inside a serving engine
 * whose allocator has already reserved the GPU's memory for its own pools,
 * or a caller with no access to an allocator at all — and so cannot hand
 * starkv_decode_attn a workspace buffer.
 *
 * Same arguments, results and error behaviour as starkv_decode_attn, minus
 * the workspace.  The scratch lives in one fixed device array inside this
 * library, STARKV_NOALLOC_SCRATCH_BYTES (32 MiB) on every GPU that loads the
 * library, kept until the process exits.  The call returns
 * STARKV_ERR_WORKSPACE, before any launch and with a message naming both
 * sizes, when starkv_workspace_bytes(layer, batch, max_pages * 16, 1) exceeds
 * that size.  That figure is the largest workspace over every decode path the
 * layer can take, so a decode that the selected path could fit in the array
 * may still be refused.  It allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 *
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.  The
 * address is kept for the life of the process: after cudaDeviceReset (or any
 * other teardown of the device's primary context) the cached address is
 * stale, so do not call this entry point again in that process.
 * Every call on a device shares the one array and leaves its contents behind;
 * each call writes every scratch element before reading it, so nothing needs
 * to start at zero.  Calls whose work overlaps on the GPU (several streams,
 * or several host threads) race on the array: serialise them.
 */
#define STARKV_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
STARKV_API starkv_status starkv_decode_attn_noalloc(const starkv_layer* layer, const void* pool, int64_t n_pages,
                                                    const int32_t* page_table, int max_pages, int batch,
                                                    const int32_t* seq_lens, const int32_t* q_pos, const void* q,
                                                    void* out, starkv_stream_t stream);

STARKV_API const char* starkv_status_string(starkv_status s);

/* Message of the last host-side error on this thread ("" if none). */
STARKV_API const char* starkv_last_error(void);

/* Library build string (version, target architecture). */
STARKV_API const char* starkv_version(void);

/*
 * Diagnostics: choose the decode implementation of a layer.
 *   0 = automatic (tensor-core kernels where the layer's shape allows them),
 *   1 = CUDA-core kernels for every step,
 *   2 = tensor-core score kernel feeding the CUDA-core value kernels.
 * Results agree within the attention tolerance; the choice exists so that each
 * implementation can be checked and timed on its own.
 */
STARKV_API starkv_status starkv_set_decode_path(starkv_layer* layer, int path);

/*
 * Measurement: per-kernel device time of the tensor-core decode, taken with
 * CUDA events recorded on the decode's own stream between its kernels (no
 * synchronisation is added to the calls).
 *   starkv_profile_decode(layer, n_calls) keeps n_calls sets of events (the
 *     next n_calls decodes fill them in order; 0 switches timing off and frees
 *     them).  Must not be called while a decode of the layer is in flight.
 *   starkv_decode_phase_ms(layer, ms, n_calls) waits for the recorded events
 *     and writes ms[c * STARKV_N_PHASES + p]: call c, phase p in the order
 *     query preparation + scores, joint values, run merge, output projection.
 *     Calls that took another decode path report zeros.
 * Returns STARKV_ERR_ARG for a NULL layer or an n_calls outside [0, 4096],
 * STARKV_ERR_CUDA if events cannot be created or read.
 */
#define STARKV_N_PHASES 4
/*
 * Diagnostics: exercise the bounded device-side wait that every pipelined
 * kernel of the decode uses, without a fault.  One CTA waits on a barrier that
 * nothing completes (no copy is issued, nobody arrives); after limit_us
 * microseconds the wait gives up, sets STARKV_DEV_TIMEOUT in the layer's
 * status word and raises the CTA's abort flag, and a second waiting role sees
 * the flag and drains, as the other roles of a decode kernel do when one
 * aborts.  No copy, MMA or tensor-memory allocation is in flight, and the CUDA
 * context stays usable: starkv_sync_status() then returns STARKV_ERR_TIMEOUT.
 * (The decode kernels' own limit is 2 seconds; "STAR-KV 阅读笔记" has no
 * counterpart, this is failure detection of the library.)
 * Returns STARKV_ERR_ARG for a NULL layer or limit_us outside [1, 2000000].
 */
STARKV_API starkv_status starkv_check_wait_timeout(const starkv_layer* layer, uint32_t limit_us,
                                                   starkv_stream_t stream);
STARKV_API starkv_status starkv_profile_decode(starkv_layer* layer, int n_calls);
STARKV_API starkv_status starkv_decode_phase_ms(const starkv_layer* layer, float* ms, int n_calls);

#ifdef __cplusplus
}
#endif

#endif /* STARKV_H */
