// Internal interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mla {

constexpr int kMaxRopePairs = 128;  // d_rope <= 256

// theta^(-2i/d_rope) for the RoPE channel pairs (host side, double precision).
inline void rope_inv_freq(double* out, int d_rope, float theta) {
  for (int i = 0; i < d_rope / 2 && i < kMaxRopePairs; ++i) out[i] = pow((double)theta, -2.0 * i / d_rope);
}

// Per-piece overhead of the tensor-core split kernel, in pages of work: loading
// the next piece's query, writing a partial and refilling the pipeline.  A clock
// trace at the v3 workload showed the workers whose chunk crossed a sequence
// start finishing ~6 % (about 7 pages of 111) after the others.
constexpr int kPairPieceCost = 8;

struct DecodeArgs {
  const uint16_t* q_lat;      // [B, nq, H, R]
  const uint16_t* pool;       // [num_pages, P, R]
  const int32_t* page_table;  // [B, max_pages]
  const int32_t* seq_lens;    // [B]
  const uint16_t* w_uv;       // [H, d_v, d_c]
  uint16_t* out;              // [B, nq, H, d_v]
  float* lse;                 // [B, nq, H] or null
  float* part_o;              // [pieces, nq*H, d_c]
  float* part_lse;            // [pieces, nq*H]
  int32_t* dev_status;        // or null
  float* out_lat;             // [B, nq, H, d_c] or null: the combine writes the merged latent
                              // output (and lse) instead of applying W_UV (context split)
  int batch, nq, n_heads, d_c, d_rope, v_head, page_size, max_pages, num_pages;
  int G;                      // split workers
  int piece_cost;             // per-piece overhead of the split kernel, in pages (plan.cuh)
  int kv_rank, kv_ranks;      // context split: this call takes window kv_rank of kv_ranks
  float scale;
};

// Partials of the ranks of a context split, merged by launch_merge_ranks: rank
// r's latent output [T, H, d_c] and lse [T, H] (device pointers: this GPU's
// memory or a peer's).
constexpr int kMaxRanks = 16;
struct RankSources {
  const float* o[kMaxRanks];
  const float* lse[kMaxRanks];
  int n;
};

struct AppendArgs {
  const uint16_t* h;          // [T, D]
  const uint16_t* w_dkv;      // [R, D]
  const int32_t* seq_idx;     // [T]
  const int32_t* pos;         // [T]
  const int32_t* page_table;  // [B, max_pages]
  uint16_t* pool;             // [num_pages, P, R]
  int32_t* dev_status;
  int n_tokens, d_model, d_c, d_rope, page_size, batch, max_pages, num_pages;
  double inv_freq[kMaxRopePairs];   // theta^(-2i/d_rope), computed on the host in double precision
};

struct AbsorbArgs {
  const uint16_t* q;          // [T, H, d_n + d_r]
  const int32_t* pos;         // [T]
  const uint16_t* w_uk;       // [H, d_n, d_c]
  uint16_t* q_lat;            // [T, H, d_c + d_r]
  int n_tokens, n_heads, qk_nope, d_c, d_rope;
  int blocks_per_cta;         // 16-token blocks each CTA of the tensor-core kernel loops over
  double inv_freq[kMaxRopePairs];
};

// y[T, N] = x[T, K] W[N, K]^T for a few tokens (the query projections, W_O)
struct LinearArgs {
  const uint16_t* x;          // [T, K]
  const uint16_t* w;          // [N, K]
  uint16_t* y;                // [T, N]
  int T, K, N;
  int ksplit;                 // CTAs of a cluster splitting K (1, 2, 4 or 8)
};

size_t decode_simt_smem_bytes(int d_c, int d_rope, int page_size);
int decode_simt_row_groups(int rows_total);
cudaError_t launch_decode_split_simt(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_combine(const DecodeArgs& a, cudaStream_t stream);
// LSE merge of the ranks' partials, then W_UV: a.batch = tokens, a.nq = 1.
cudaError_t launch_merge_ranks(const DecodeArgs& a, const RankSources& src, cudaStream_t stream);

// 2-D TMA map over bf16 rows of 576 elements (row stride 1152 bytes) with a box
// of [box_rows x box_cols] elements (tma_map.cu).
bool encode_rows576(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                    CUtensorMapSwizzle sw);

// Tensor-core split kernel on CTA pairs (d_c = 512, d_rope = 64, 64-token pages).
bool decode_pair_supported(int d_c, int d_rope, int page_size);
// Split workers (CTA pairs) per 128-row tile when every tile gets its own set.
int decode_pair_workers(int sms, int rows_total);
cudaError_t launch_decode_split_pair(const DecodeArgs& a, long long spin_limit, cudaStream_t stream);
constexpr long long kSpinLimitCycles = 1ll << 31;  // ~1 s at B200 clocks per bounded wait

// Launch attribute that lets a kernel start while its predecessor on the stream
// finishes (every kernel of this library waits for the predecessor, with
// griddepcontrol.wait, before it reads any input).
inline cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at.val.programmaticStreamSerializationAllowed = 1;
  return at;
}
// MLA_OK for cudaSuccess; otherwise remembers `e` for mla_last_cuda_error (per host
// thread) and returns MLA_ERR_CUDA (api.cu).
int record_cuda_error(cudaError_t e);

cudaError_t launch_append_latent(const AppendArgs& a, cudaStream_t stream);
cudaError_t launch_absorb_q(const AbsorbArgs& a, cudaStream_t stream);
// Both of the above in one launch when the token count allows (<= 16 tokens),
// else the two launches in turn.
cudaError_t launch_append_absorb(const AppendArgs& ap, const AbsorbArgs& ab, cudaStream_t stream);
int linear_ksplit(int N, int K, int sms);
cudaError_t launch_linear(const LinearArgs& a, cudaStream_t stream);

}  // namespace mla
