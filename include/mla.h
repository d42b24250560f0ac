/*
 * mla.h - C ABI of the B200 (sm_100a) absorbed Multi-Head Latent Attention
 * decode library (libmla_b200.so).
 *
 * One decode step of one attention layer is three calls, in this order:
 *   mla_append_latent  write this step's latent-cache rows [c_t || k_t^R]
 *   mla_absorb_q       fold W_UK into the queries, rotate their RoPE part
 *   mla_decode_attn    split-KV attention over the paged latent cache,
 *                      log-sum-exp combine of the splits, then W_UV
 * Around them: mla_query_proj (the queries from the hidden state through the
 * compressed query latent, before mla_absorb_q) and mla_out_proj (the layer
 * output W_O concat_h(o_h), after mla_decode_attn).  For sequences too long
 * for one GPU, mla_decode_attn_partial (one rank's window of the pages) and
 * mla_merge_ranks (the ranks' partials merged, then W_UV) split the key range.
 * Keys and values are never decompressed: every cached token holds only its
 * latent c_t (d_c scalars) and its decoupled RoPE key k_t^R (d_rope scalars).
 *
 * Sources (page title, section):
 *   [eyestech-pypi]  "eyestech-mla 1.0.0" package description: "Key Architectural
 *                    Highlights" (576 = 512 + 64 scalars per token; query
 *                    absorption), quickstart "Autoregressive MLA Decoding with
 *                    Query Absorption" (decode step appends to the cache, 1024 -> 1025).
 *   [eyestech-blog]  "DeepSeek MLA Architecture: How It Cuts KV Cache by 93%",
 *                    sec. 2 "Query Matrix Absorption" (q~ = W_UK^T q).
 *   [from-scratch]   "mla-from-scratch" README, "Absorption, and why RoPE breaks it"
 *                    (content + positional score; W_UV applied once after attending
 *                    over latents; refuse to build without decoupled RoPE).
 *   [distaisys]      "Deep-Dive: Multi-Head Latent Attention (MLA) and Low-Rank KV
 *                    Cache Compression in DeepSeek-V3", sec. 2 (c = W_DKV h,
 *                    k = W_UK c, v = W_UV c) and sec. 3 (weight layouts, softmax).
 *   [songhuiming]    "MHA vs MLA KV cache comparison", "MLA ... Step-by-step for
 *                    t100" (append the new latent, then attend over all of them).
 *
 * Conventions shared by every call
 *   - Tensors are dense, row-major (last index fastest), on the current CUDA
 *     device unless stated.  "bf16" buffers hold IEEE bfloat16 bit patterns.
 *   - Every device pointer must be 16-byte aligned (MLA_ERR_MISALIGNED).
 *   - The caller owns every buffer.  The library allocates no device or host
 *     memory and keeps no state between calls, with one exception:
 *     mla_decode_attn_noalloc works in a fixed scratch array the library
 *     defines in device memory (a static __device__ array, not an allocation)
 *     and caches that array's address per device (see its declaration).  Calls
 *     are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream).
 *   - Host-checkable errors return a negative mla_status before anything is
 *     launched.  Errors only the device can see (a page id outside the pool, a
 *     sequence length outside the page table, a bounded wait that ran out) are
 *     recorded, first one wins, in the caller's int32 status word `dev_status`
 *     (may be NULL) and the offending access is skipped: no kernel traps.
 *   - Bounded waits: each wait between the roles of the decode kernels gives up
 *     after about 2^31 cycles (~1 s), records MLA_ERR_TIMEOUT and ends the kernel
 *     cleanly.  The environment variable MLA_SPIN_LIMIT (cycles, read at each
 *     call) overrides the budget; tests set it small to exercise that path.
 *   - Overlap with the preceding kernel: every kernel is launched with
 *     programmatic dependent launch and may start while the kernel enqueued
 *     just before it on `stream` finishes.  Activations, caches, page tables
 *     and lengths are read only after waiting for that kernel; weight matrices
 *     (w_dkv, w_uk, w_uv, w_o, w_dq, w_uq) may be read before, so the kernel
 *     enqueued immediately before a call must not write a weight that the call
 *     reads (any earlier work on the stream may).
 *   - RoPE: channel pair (2i, 2i+1) rotates by pos * theta^(-2i/d_rope), the
 *     angle evaluated in double precision; pos = cache index of the token.
 *   - bf16 outputs are rounded to nearest even from fp32 accumulators.
 */
#ifndef MLA_B200_H_
#define MLA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t mla_bf16; /* bfloat16 bit pattern */

/* Layer dimensions.  Names follow the pages: d_c = kv_lora_rank (latent width),
 * d_rope = decoupled RoPE width (qk_rope_dim), qk_nope = per-head non-rotary
 * query/key width d_h, v_head = per-head value width, d_model = D. */
typedef struct mla_dims {
  int32_t n_heads;      /* H, 1..128 */
  int32_t d_c;          /* multiple of 8 */
  int32_t d_rope;       /* even, multiple of 8, > 0: absorption needs decoupled RoPE */
  int32_t qk_nope;      /* multiple of 8 */
  int32_t v_head;       /* multiple of 8 */
  int32_t d_model;      /* multiple of 8 */
  int32_t page_size;    /* tokens per latent-cache page: 64 */
  float softmax_scale;  /* 0 selects 1/sqrt(qk_nope + d_rope) */
  float rope_theta;     /* 0 selects 10000 */
} mla_dims;

typedef enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1,  /* NULL pointer, non-positive size, bad count */
  MLA_ERR_UNSUPPORTED = -2,  /* dimensions this build does not implement */
  MLA_ERR_MISALIGNED = -3,   /* a pointer is not 16-byte aligned */
  MLA_ERR_WORKSPACE = -4,    /* workspace smaller than mla_decode_workspace_bytes */
  MLA_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed */
  MLA_ERR_TIMEOUT = -6,      /* device: a bounded wait inside a kernel ran out */
  MLA_ERR_RANGE = -7         /* device: page id / position / length out of range */
} mla_status;

/*
 * mla_append_latent - write this step's latent-cache rows.
 *
 * For each token t (0 <= t < n_tokens) with hidden state h[t] (length d_model):
 *   [c_t || k^_t] = w_dkv h[t]          c_t = W_DKV h_t ([distaisys] sec. 2),
 *                                       k^_t = W_KR h_t (the RoPE key projection)
 *   k_t^R = RoPE(k^_t, pos[t])          decoupled RoPE key ([eyestech-pypi] item 2)
 *   pool[page_table[seq_idx[t]][pos[t] / page]][pos[t] % page][:] = bf16([c_t || k_t^R])
 * fp32 accumulation, one bf16 rounding per stored element.
 *
 *   h          device bf16 [n_tokens, d_model]
 *   w_dkv      device bf16 [d_c + d_rope, d_model]; rows 0..d_c-1 = W_DKV, the rest W_KR
 *   seq_idx    device int32 [n_tokens], each in [0, batch)
 *   pos        device int32 [n_tokens], cache index = RoPE position, in [0, max_pages*page)
 *   page_table device int32 [batch, max_pages]; physical page ids in [0, num_pages)
 *   pool       device bf16 [num_pages, page_size, d_c + d_rope] (written in place)
 *   dev_status device int32 word or NULL; device-side range errors land here
 * Two tokens writing the same slot race (the caller must not do that).
 * Returns MLA_OK or a negative mla_status.  n_tokens == 0 is a no-op.
 */
int mla_append_latent(const mla_dims* dims, const mla_bf16* h, const mla_bf16* w_dkv,
                      const int32_t* seq_idx, const int32_t* pos, const int32_t* page_table,
                      int32_t batch, int32_t max_pages, mla_bf16* pool, int32_t num_pages,
                      int32_t n_tokens, int32_t* dev_status, void* stream);

/*
 * mla_absorb_q - absorbed queries.
 *
 * For each token t and head h, with q[t][h] = [q_nope (qk_nope) || q_rope (d_rope)]:
 *   q_lat[t][h][0 : d_c]        = W_UK,h^T q_nope   ([eyestech-blog] sec. 2;
 *                                 [from-scratch] "Absorption, and why RoPE breaks it")
 *   q_lat[t][h][d_c : d_c+d_rope] = RoPE(q_rope, pos[t])
 * so that q_nope . (W_UK,h c) = q_lat[0:d_c] . c for every cached latent c.
 *
 *   q      device bf16 [n_tokens, H, qk_nope + d_rope]
 *   pos    device int32 [n_tokens]; the query's own cache index (>= 0)
 *   w_uk   device bf16 [H, qk_nope, d_c]   (w_uk[h] = W_UK,h, maps c to a key head)
 *   q_lat  device bf16 [n_tokens, H, d_c + d_rope] (output)
 * fp32 accumulation, bf16 output.  n_tokens == 0 is a no-op.
 */
int mla_absorb_q(const mla_dims* dims, const mla_bf16* q, const int32_t* pos,
                 const mla_bf16* w_uk, mla_bf16* q_lat, int32_t n_tokens, void* stream);

/*
 * mla_append_absorb - mla_append_latent and mla_absorb_q of one decode step in
 * one call: the step's n_tokens tokens are appended (h, w_dkv, seq_idx, pos,
 * page_table, pool as in mla_append_latent) and their queries absorbed (q, w_uk,
 * q_lat as in mla_absorb_q, with the same pos: a decode token's query sits at
 * the cache index of the row it appends).  The two computations are
 * independent ([songhuiming] "Step-by-step for t100": the new latent is
 * appended and the query absorbed before attending); with n_tokens <= 16 they
 * run in one kernel launch, so neither waits for the other, else as the two
 * calls in turn.  Results equal those of the two calls up to the order of the
 * fp32 sums of the append (q_lat bit for bit).  Arguments, errors and the
 * device status word as in the two calls; n_tokens == 0 is a no-op.
 */
int mla_append_absorb(const mla_dims* dims, const mla_bf16* h, const mla_bf16* w_dkv,
                      const int32_t* seq_idx, const int32_t* pos, const int32_t* page_table,
                      int32_t batch, int32_t max_pages, mla_bf16* pool, int32_t num_pages,
                      const mla_bf16* q, const mla_bf16* w_uk, mla_bf16* q_lat, int32_t n_tokens,
                      int32_t* dev_status, void* stream);

/*
 * mla_decode_workspace_bytes - device workspace mla_decode_attn needs for
 * `batch` sequences with `nq` query tokens each, on the current device.
 * Returns 0 for invalid arguments.
 */
size_t mla_decode_workspace_bytes(const mla_dims* dims, int32_t batch, int32_t nq);

/*
 * mla_decode_attn - absorbed latent attention over the paged cache, then W_UV.
 *
 * Query token i (0 <= i < nq) of sequence b sits at cache index
 * p = seq_lens[b] - nq + i and attends to cache indices 0..p (its own row, already
 * appended, included; later tokens of the same step masked).  For head h with
 * q_lat row [q~ || q_r] and cache row n = [c_n || k_n^R]:
 *   s_n   = scale * (q~ . c_n + q_r . k_n^R)       content + positional score
 *                                                  ([from-scratch], same section)
 *   p     = softmax(s)                             scale = dims->softmax_scale or
 *                                                  1/sqrt(qk_nope + d_rope)
 *   o_lat = sum_n p_n c_n                          values read in latent space
 *   out[b][i][h] = W_UV,h o_lat                    up-projected once ([from-scratch])
 *   lse[b][i][h] = log sum_n exp(s_n)              natural log
 * The key range of every sequence is cut into pages processed in parallel
 * (split-KV); each part's softmax-normalised o_lat and lse go to the workspace
 * and a combine step merges them with weights exp(lse_part - lse).
 *
 *   q_lat      device bf16 [batch, nq, H, d_c + d_rope] (as written by mla_absorb_q)
 *   pool       device bf16 [num_pages, page_size, d_c + d_rope]
 *   page_table device int32 [batch, max_pages]
 *   seq_lens   device int32 [batch]: cache length after this step's append,
 *              nq <= seq_lens[b] <= max_pages * page_size
 *   w_uv       device bf16 [H, v_head, d_c]   (w_uv[h] = W_UV,h)
 *   workspace  device scratch of ws_bytes >= mla_decode_workspace_bytes(...)
 *   out        device bf16 [batch, nq, H, v_head] (output)
 *   lse        device fp32 [batch, nq, H] (output) or NULL
 *   dev_status device int32 word or NULL
 * A sequence whose length is out of range gets zero output and lse = -inf; a
 * page-table entry outside [0, num_pages) is skipped (never read).  Both record
 * MLA_ERR_RANGE in dev_status.  batch <= 1024, nq <= 1024, batch * nq <= 2^18
 * (else MLA_ERR_UNSUPPORTED).  nq > 1 covers decode with several new tokens per
 * sequence and chunked prefill: a chunk of nq new tokens, appended by
 * mla_append_latent first, attends causally (token i of the chunk sees the cache
 * up to its own index).  Each group of 128 query rows (token, head) streams the
 * sequence's pages once.
 */
int mla_decode_attn(const mla_dims* dims, const mla_bf16* q_lat, const mla_bf16* pool,
                    const int32_t* page_table, const int32_t* seq_lens, int32_t batch,
                    int32_t nq, int32_t max_pages, int32_t num_pages, const mla_bf16* w_uv,
                    void* workspace, size_t ws_bytes, mla_bf16* out, float* lse,
                    int32_t* dev_status, void* stream);

/*
 * mla_decode_attn_partial - one rank's share of a context-split decode.
 *
 * For a sequence too long for one GPU the key range is split over kv_ranks
 * ranks (one call per rank, normally one rank per GPU): rank r attends over the
 * pages [P_b r / R, P_b (r + 1) / R) of each sequence's P_b = ceil(seq_lens[b] /
 * page_size) pages (R = kv_ranks), with the masking of mla_decode_attn (absolute
 * key indices), and writes its softmax-normalised latent output and log-sum-exp:
 *   o_lat[b][i][h][:] = sum_{n in window} p_n c_n / sum_{n in window} p_n
 *   lse[b][i][h]      = log sum_{n in window} exp(s_n)   (-inf for an empty window)
 * mla_merge_ranks then merges the ranks' results.  This is split-KV across
 * GPUs: the partials are the only data the ranks exchange (d_c + 1 floats per
 * query row and rank).  kv_ranks = 1 gives the whole cache.
 *
 *   o_lat  device fp32 [batch, nq, H, d_c] (output)
 *   lse    device fp32 [batch, nq, H] (output)
 *   other arguments as for mla_decode_attn (no W_UV: it is applied by the merge).
 * 0 <= kv_rank < kv_ranks, else MLA_ERR_INVALID_ARG.
 */
int mla_decode_attn_partial(const mla_dims* dims, const mla_bf16* q_lat, const mla_bf16* pool,
                            const int32_t* page_table, const int32_t* seq_lens, int32_t batch, int32_t nq,
                            int32_t max_pages, int32_t num_pages, int32_t kv_rank, int32_t kv_ranks,
                            void* workspace, size_t ws_bytes, float* o_lat, float* lse, int32_t* dev_status,
                            void* stream);

/*
 * mla_merge_ranks - merge the ranks' partials of a context-split decode, then W_UV.
 *
 * For each query row (token t, head h), with rank r's partial (o_r, lse_r):
 *   LSE = log sum_r exp(lse_r),  o_lat = sum_r exp(lse_r - LSE) o_r
 *   out[t][h] = W_UV,h o_lat,  lse_out[t][h] = LSE
 * the same log-sum-exp merge as the split-KV combine inside mla_decode_attn.
 *
 *   o_lat    host array of n_ranks device pointers, each to fp32 [n_tokens, H, d_c]
 *   lse      host array of n_ranks device pointers, each to fp32 [n_tokens, H]
 *   w_uv     device bf16 [H, v_head, d_c]
 *   out      device bf16 [n_tokens, H, v_head] (output)
 *   lse_out  device fp32 [n_tokens, H] (output) or NULL
 * The partials are read with plain loads, once each: a pointer may address this
 * GPU's memory or a peer GPU's memory mapped into this process (NVLink peer
 * access), so the exchange between the ranks happens inside this kernel.
 * 1 <= n_ranks <= 16, n_tokens <= 2^18 (else MLA_ERR_UNSUPPORTED); n_tokens == 0
 * is a no-op.
 */
int mla_merge_ranks(const mla_dims* dims, const float* const* o_lat, const float* const* lse, int32_t n_ranks,
                    int32_t n_tokens, const mla_bf16* w_uv, mla_bf16* out, float* lse_out, void* stream);

/*
 * mla_decode_attn_noalloc - mla_decode_attn for callers that cannot allocate.
 *
 * The pages describe no such call; it exists for deployment.  Some callers
 * cannot give mla_decode_attn a workspace: code that runs inside a host framework
 * which owns all device memory (a serving-engine plugin with a fixed memory
 * budget, where only the framework allocates), or a latency-critical decode loop
 * that must not call cudaMalloc because it can synchronise the device.  This call
 * computes exactly what mla_decode_attn computes (same arguments minus the
 * workspace) and allocates nothing: no cudaMalloc, no cudaFree, no allocating
 * library routine.
 *
 * Scratch: a 64 MiB device array owned by the library.  Every GPU that loads the
 * library holds one copy until the process exits.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress) with that device
 * current; make that first call before any stream capture.
 * Limit: a call whose mla_decode_workspace_bytes(dims, batch, nq) exceeds 64 MiB
 * returns MLA_ERR_WORKSPACE without launching anything.
 * Sharing: all calls on a device use the same array, which keeps the last call's
 * contents.  Nothing in it needs to start at zero.  Calls that overlap on the GPU
 * (on different streams, or from several host threads) race on the array and
 * corrupt each other's results: issue them one after another on one stream.
 * Other arguments, outputs and errors: as for mla_decode_attn.
 */
int mla_decode_attn_noalloc(const mla_dims* dims, const mla_bf16* q_lat, const mla_bf16* pool,
                            const int32_t* page_table, const int32_t* seq_lens, int32_t batch,
                            int32_t nq, int32_t max_pages, int32_t num_pages, const mla_bf16* w_uv,
                            mla_bf16* out, float* lse, int32_t* dev_status, void* stream);

/*
 * mla_out_proj - layer output projection of the step's tokens.
 *
 * For each token t and output feature i (0 <= i < d_model):
 *   y[t][i] = sum_{h < H, j < v_head} w_o[i][h * v_head + j] * o[t][h][j]
 * i.e. y = W_O concat_h(o_h), the heads' outputs concatenated head after head
 * ([distaisys] sec. 3, out_proj of width H * d_h -> d_model, no bias).  Because
 * mla_decode_attn applies W_UV once after attending over the latents, W_UV and
 * W_O act back to back here ([from-scratch] "Absorption, and why RoPE breaks it":
 * they fold into one matrix by associativity); this call keeps them separate so
 * that `o` stays available per head.
 *
 *   o     device bf16 [n_tokens, H, v_head]; the `out` of mla_decode_attn
 *         ([batch, nq, H, v_head]) with n_tokens = batch * nq
 *   w_o   device bf16 [d_model, H * v_head]
 *   y     device bf16 [n_tokens, d_model] (output; must not overlap o or w_o)
 * fp32 accumulation, one bf16 rounding per output.  n_tokens == 0 is a no-op;
 * n_tokens > 2^20 returns MLA_ERR_UNSUPPORTED.  The weight is streamed once per
 * 32 tokens (once per call for n_tokens <= 32).
 */
int mla_out_proj(const mla_dims* dims, const mla_bf16* o, const mla_bf16* w_o, mla_bf16* y,
                 int32_t n_tokens, void* stream);

/*
 * mla_query_proj - queries through the compressed query latent (q-LoRA).
 *
 * For each token t:
 *   c_q[t] = bf16(W_DQ h[t])               width q_lora_rank (1536 in the V3-shaped
 *                                          decoder of [eyestech-blog] sec. 3)
 *   q[t]   = bf16(W_UQ c_q[t]) as [H][qk_nope + d_rope], per head q_nope then q_rope
 * ([songhuiming] "Note on Actual Implementation": the query side is down- then
 * up-projected).  The pages name no normalisation between the two maps; none is
 * applied.  c_q is rounded to bf16 before the up-projection (a bf16 module's
 * activation) and is returned.  q is the input of mla_absorb_q (RoPE not applied).
 *
 *   h     device bf16 [n_tokens, d_model]
 *   w_dq  device bf16 [q_lora_rank, d_model]
 *   w_uq  device bf16 [H * (qk_nope + d_rope), q_lora_rank]; rows head-major
 *   c_q   device bf16 [n_tokens, q_lora_rank] (output)
 *   q     device bf16 [n_tokens, H, qk_nope + d_rope] (output)
 * fp32 accumulation.  q_lora_rank must be a multiple of 8 (<= 65536); n_tokens ==
 * 0 is a no-op; n_tokens > 2^20 returns MLA_ERR_UNSUPPORTED.  Outputs must not
 * overlap the inputs.  Two kernels, in order, on `stream`.
 */
int mla_query_proj(const mla_dims* dims, int32_t q_lora_rank, const mla_bf16* h, const mla_bf16* w_dq,
                   const mla_bf16* w_uq, mla_bf16* c_q, mla_bf16* q, int32_t n_tokens, void* stream);

/* mla_status_read - wait for `stream`, then return the mla_status recorded in the
 * device word dev_status (MLA_OK if none), or MLA_ERR_CUDA if the copy failed. */
int mla_status_read(const int32_t* dev_status, void* stream);

/* mla_status_clear - reset the device word to MLA_OK (asynchronous on stream). */
int mla_status_clear(int32_t* dev_status, void* stream);

/* mla_last_cuda_error - the CUDA runtime error code behind the last MLA_ERR_CUDA
 * returned to the calling host thread (0 if none); *name (if name is not NULL)
 * receives its static name, e.g. "cudaErrorLaunchOutOfResources". */
int mla_last_cuda_error(const char** name);

/* mla_status_string - static description of an mla_status value. */
const char* mla_status_string(int status);

/* mla_version - library version string, e.g. "mla_b200 0.1.0 sm_100a". */
const char* mla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H_ */
