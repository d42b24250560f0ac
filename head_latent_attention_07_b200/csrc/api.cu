// C ABI of libmla_b200.so: argument validation, workspace sizing, launches.
// The declarations and the contract of every entry point are in include/mla.h.
#include <math.h>
#include <stdlib.h>

#include "../../include/mla.h"
#include "decode.h"
#include "plan.cuh"

namespace {

constexpr float kDefaultTheta = 10000.f;
constexpr int32_t kMaxOutProjTokens = 1 << 20;   // tokens of one out / query projection call
constexpr int32_t kMaxQLoraRank = 1 << 16;
constexpr int32_t kMaxMergeTokens = 1 << 18;     // grid rows of the rank merge stay below 65536
// Query tokens per sequence of one decode call: 1 or 2 in decode, up to a
// chunk of 1024 in chunked prefill; batch * nq is bounded like the merge's tokens.
constexpr int32_t kMaxNq = 1024;
bool decode_shape_ok(int32_t batch, int32_t nq) {
  return batch <= mla::kMaxBatch && nq <= kMaxNq && (int64_t)batch * nq <= kMaxMergeTokens;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Spin budget of each bounded wait in the split kernel: kSpinLimitCycles, or the
// environment variable MLA_SPIN_LIMIT (cycles, >= 0) when it is set, which lets a
// test make the waits run out.
long long spin_limit_cycles() {
  const char* e = getenv("MLA_SPIN_LIMIT");
  if (e != nullptr && *e != 0) {
    char* end = nullptr;
    const long long v = strtoll(e, &end, 10);
    if (end != nullptr && *end == 0 && v >= 0) return v;
  }
  return mla::kSpinLimitCycles;
}

// Shape checks shared by all calls.  d_rope == 0 is refused: without the
// decoupled RoPE channels W_UK cannot be folded into the query (the rotation
// sits between W_Q and W_UK), so an "absorbed" result would be wrong.
int check_dims(const mla_dims* d) {
  if (d == nullptr) return MLA_ERR_INVALID_ARG;
  if (d->n_heads < 1 || d->d_c < 1 || d->qk_nope < 1 || d->v_head < 1 || d->d_model < 1 ||
      d->page_size < 1 || d->d_rope < 0)
    return MLA_ERR_INVALID_ARG;
  if (d->d_rope == 0) return MLA_ERR_UNSUPPORTED;
  if (d->n_heads > 128 || d->d_c > 512 || d->d_c % 8 || d->d_rope % 8 || d->d_rope > 256 ||
      d->qk_nope % 8 || d->qk_nope > 1024 || d->v_head % 8 || d->v_head > 1024 ||
      d->d_model % 8 || d->page_size > 256)
    return MLA_ERR_UNSUPPORTED;
  // one cache page and the query rows of a CTA must fit in shared memory
  if (mla::decode_simt_smem_bytes(d->d_c, d->d_rope, d->page_size) > 200 * 1024) return MLA_ERR_UNSUPPORTED;
  if (!(d->softmax_scale >= 0.f) || isinf(d->softmax_scale) || !(d->rope_theta >= 0.f) ||
      isinf(d->rope_theta))
    return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

float eff_scale(const mla_dims* d) {
  return d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / sqrtf((float)(d->qk_nope + d->d_rope));
}
float eff_theta(const mla_dims* d) { return d->rope_theta > 0.f ? d->rope_theta : kDefaultTheta; }

int cuda_status(cudaError_t e);

int device_sms(int* sms) {
  int dev = 0;
  int st = cuda_status(cudaGetDevice(&dev));
  if (st != MLA_OK) return st;
  return cuda_status(cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev));
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  size_t part_o_bytes, part_lse_bytes, total;
};

// Split workers of a decode call: one CTA pair per worker and 128-row tile on the
// tensor-core path (fewer workers when there are many row tiles, as in chunked
// prefill), else a share of two CTAs per SM over the 16-row groups.
int decode_workers(const mla_dims* d, int nq, int sms) {
  if (mla::decode_pair_supported(d->d_c, d->d_rope, d->page_size)) {
    const int tiles = (nq * d->n_heads + 127) / 128;
    const int pairs = sms / 2;
    const int g_decode = mla::decode_pair_workers(sms, nq * d->n_heads);
    if (g_decode > 1) return g_decode;   // few row tiles (decode): one wave of pairs
    // many row tiles (chunked prefill): split each tile's pages over G workers,
    // G <= 8 chosen so that the last wave of CTA pairs is as full as possible
    int best = 1;
    double best_fill = 0.0;
    for (int g = 1; g <= 8; ++g) {
      const long long units = (long long)tiles * g;
      const double fill = (double)units / (double)(((units + pairs - 1) / pairs) * pairs);
      if (fill > best_fill + 1e-9) { best_fill = fill; best = g; }
    }
    return best;
  }
  const int groups = mla::decode_simt_row_groups(nq * d->n_heads);
  const int G = (2 * sms + groups - 1) / groups;
  return G < 1 ? 1 : (G > sms ? sms : G);
}

// Workspace for at most (workers + batch) split pieces of nq*H rows each.
WsLayout ws_layout(const mla_dims* d, int batch, int nq, int sms) {
  const size_t pieces = (size_t)mla::max_pieces(decode_workers(d, nq, sms), batch);
  const size_t rows = (size_t)nq * d->n_heads;
  WsLayout w;
  w.part_o_bytes = align256(pieces * rows * d->d_c * sizeof(float));
  w.part_lse_bytes = align256(pieces * rows * sizeof(float));
  w.total = w.part_o_bytes + w.part_lse_bytes;
  return w;
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;  // per calling host thread

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MLA_OK;
  g_last_cuda_error = e;
  return MLA_ERR_CUDA;
}

}  // namespace

namespace mla {
int record_cuda_error(cudaError_t e) { return cuda_status(e); }
}  // namespace mla

namespace {

// Checks and fills the arguments of mla_append_latent (also for mla_append_absorb).
int append_args(const mla_dims* dims, const mla_bf16* h, const mla_bf16* w_dkv, const int32_t* seq_idx,
                const int32_t* pos, const int32_t* page_table, int32_t batch, int32_t max_pages, mla_bf16* pool,
                int32_t num_pages, int32_t n_tokens, int32_t* dev_status, mla::AppendArgs* a) {
  int st = check_dims(dims);
  if (st != MLA_OK) return st;
  if (n_tokens < 0 || batch < 1 || max_pages < 1 || num_pages < 1) return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  if (!h || !w_dkv || !seq_idx || !pos || !page_table || !pool) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_dkv) || !aligned16(seq_idx) || !aligned16(pos) ||
      !aligned16(page_table) || !aligned16(pool) || (dev_status && !aligned16(dev_status)))
    return MLA_ERR_MISALIGNED;
  if ((int64_t)max_pages * dims->page_size > INT32_MAX) return MLA_ERR_UNSUPPORTED;
  a->h = h; a->w_dkv = w_dkv; a->seq_idx = seq_idx; a->pos = pos; a->page_table = page_table;
  a->pool = pool; a->dev_status = dev_status; a->n_tokens = n_tokens; a->d_model = dims->d_model;
  a->d_c = dims->d_c; a->d_rope = dims->d_rope; a->page_size = dims->page_size; a->batch = batch;
  a->max_pages = max_pages; a->num_pages = num_pages;
  mla::rope_inv_freq(a->inv_freq, dims->d_rope, eff_theta(dims));
  return MLA_OK;
}

// Checks and fills the arguments of mla_absorb_q (also for mla_append_absorb).
int absorb_args(const mla_dims* dims, const mla_bf16* q, const int32_t* pos, const mla_bf16* w_uk,
                mla_bf16* q_lat, int32_t n_tokens, mla::AbsorbArgs* a) {
  int st = check_dims(dims);
  if (st != MLA_OK) return st;
  if (n_tokens < 0) return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  if (!q || !pos || !w_uk || !q_lat) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(pos) || !aligned16(w_uk) || !aligned16(q_lat)) return MLA_ERR_MISALIGNED;
  a->q = q; a->pos = pos; a->w_uk = w_uk; a->q_lat = q_lat; a->n_tokens = n_tokens;
  a->n_heads = dims->n_heads; a->qk_nope = dims->qk_nope; a->d_c = dims->d_c; a->d_rope = dims->d_rope;
  // each CTA stages one head's W_UK (one CTA per SM fits) and loops over a run of
  // 16-token blocks: as many CTAs per head as fit in one wave, so that W_UK is
  // read about once per such CTA instead of once per block
  int sms = 0;
  if ((st = device_sms(&sms)) != MLA_OK) return st;
  const int blocks = (n_tokens + 15) / 16;
  int per_head = sms / dims->n_heads;
  if (per_head < 1) per_head = 1;
  a->blocks_per_cta = (blocks + per_head - 1) / per_head;
  mla::rope_inv_freq(a->inv_freq, dims->d_rope, eff_theta(dims));
  return MLA_OK;
}

}  // namespace


extern "C" {

int mla_append_latent(const mla_dims* dims, const mla_bf16* h, const mla_bf16* w_dkv,
                      const int32_t* seq_idx, const int32_t* pos, const int32_t* page_table,
                      int32_t batch, int32_t max_pages, mla_bf16* pool, int32_t num_pages,
                      int32_t n_tokens, int32_t* dev_status, void* stream) {
  mla::AppendArgs a;
  const int st = append_args(dims, h, w_dkv, seq_idx, pos, page_table, batch, max_pages, pool, num_pages, n_tokens,
                             dev_status, &a);
  if (st != MLA_OK || n_tokens == 0) return st;
  return cuda_status(mla::launch_append_latent(a, (cudaStream_t)stream));
}

int mla_absorb_q(const mla_dims* dims, const mla_bf16* q, const int32_t* pos,
                 const mla_bf16* w_uk, mla_bf16* q_lat, int32_t n_tokens, void* stream) {
  mla::AbsorbArgs a;
  const int st = absorb_args(dims, q, pos, w_uk, q_lat, n_tokens, &a);
  if (st != MLA_OK || n_tokens == 0) return st;
  return cuda_status(mla::launch_absorb_q(a, (cudaStream_t)stream));
}

int mla_append_absorb(const mla_dims* dims, const mla_bf16* h, const mla_bf16* w_dkv, const int32_t* seq_idx,
                      const int32_t* pos, const int32_t* page_table, int32_t batch, int32_t max_pages,
                      mla_bf16* pool, int32_t num_pages, const mla_bf16* q, const mla_bf16* w_uk,
                      mla_bf16* q_lat, int32_t n_tokens, int32_t* dev_status, void* stream) {
  mla::AppendArgs ap;
  mla::AbsorbArgs ab;
  int st = append_args(dims, h, w_dkv, seq_idx, pos, page_table, batch, max_pages, pool, num_pages, n_tokens,
                       dev_status, &ap);
  if (st != MLA_OK) return st;
  if ((st = absorb_args(dims, q, pos, w_uk, q_lat, n_tokens, &ab)) != MLA_OK || n_tokens == 0) return st;
  return cuda_status(mla::launch_append_absorb(ap, ab, (cudaStream_t)stream));
}

size_t mla_decode_workspace_bytes(const mla_dims* dims, int32_t batch, int32_t nq) {
  if (check_dims(dims) != MLA_OK || batch < 1 || nq < 1 || !decode_shape_ok(batch, nq)) return 0;
  int sms = 0;
  if (device_sms(&sms) != MLA_OK) return 0;
  return ws_layout(dims, batch, nq, sms).total;
}

}  // extern "C"

namespace {

// The decode path of mla_decode_attn (out set) and mla_decode_attn_partial
// (o_lat set: the combine writes the merged latent output of this rank's window).
int decode_common(const mla_dims* dims, const mla_bf16* q_lat, const mla_bf16* pool, const int32_t* page_table,
                  const int32_t* seq_lens, int32_t batch, int32_t nq, int32_t max_pages, int32_t num_pages,
                  const mla_bf16* w_uv, int32_t kv_rank, int32_t kv_ranks, void* workspace, size_t ws_bytes,
                  mla_bf16* out, float* o_lat, float* lse, int32_t* dev_status, void* stream) {
  int st = check_dims(dims);
  if (st != MLA_OK) return st;
  if (batch < 1 || nq < 1 || max_pages < 1 || num_pages < 1) return MLA_ERR_INVALID_ARG;
  if (kv_ranks < 1 || kv_rank < 0 || kv_rank >= kv_ranks) return MLA_ERR_INVALID_ARG;
  if (!decode_shape_ok(batch, nq)) return MLA_ERR_UNSUPPORTED;
  if ((int64_t)max_pages * dims->page_size > INT32_MAX) return MLA_ERR_UNSUPPORTED;
  if (!q_lat || !pool || !page_table || !seq_lens || !workspace || (!out && !o_lat)) return MLA_ERR_INVALID_ARG;
  if (out && !w_uv) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_lat) || !aligned16(pool) || !aligned16(page_table) || !aligned16(seq_lens) ||
      (w_uv && !aligned16(w_uv)) || !aligned16(workspace) || (out && !aligned16(out)) ||
      (o_lat && !aligned16(o_lat)) || (lse && !aligned16(lse)) || (dev_status && !aligned16(dev_status)))
    return MLA_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_sms(&sms)) != MLA_OK) return st;
  const WsLayout wl = ws_layout(dims, batch, nq, sms);
  if (ws_bytes < wl.total) return MLA_ERR_WORKSPACE;

  mla::DecodeArgs a;
  a.q_lat = q_lat; a.pool = pool; a.page_table = page_table; a.seq_lens = seq_lens; a.w_uv = w_uv;
  a.out = out; a.lse = lse; a.dev_status = dev_status; a.out_lat = o_lat;
  a.part_o = reinterpret_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + wl.part_o_bytes);
  a.batch = batch; a.nq = nq; a.n_heads = dims->n_heads; a.d_c = dims->d_c; a.d_rope = dims->d_rope;
  a.v_head = dims->v_head; a.page_size = dims->page_size; a.max_pages = max_pages;
  a.num_pages = num_pages; a.scale = eff_scale(dims);
  a.kv_rank = kv_rank; a.kv_ranks = kv_ranks;
  cudaStream_t s = (cudaStream_t)stream;
  a.G = decode_workers(dims, nq, sms);
  const bool pair = mla::decode_pair_supported(dims->d_c, dims->d_rope, dims->page_size);
  a.piece_cost = pair ? mla::kPairPieceCost : 0;
  if (pair) {
    // tensor-core path: one CTA pair per worker and 128-row tile
    if ((st = cuda_status(mla::launch_decode_split_pair(a, spin_limit_cycles(), s))) != MLA_OK) return st;
  } else {
    if ((st = cuda_status(mla::launch_decode_split_simt(a, s))) != MLA_OK) return st;
  }
  return cuda_status(mla::launch_decode_combine(a, s));
}

}  // namespace

extern "C" {

int mla_decode_attn(const mla_dims* dims, const mla_bf16* q_lat, const mla_bf16* pool,
                    const int32_t* page_table, const int32_t* seq_lens, int32_t batch,
                    int32_t nq, int32_t max_pages, int32_t num_pages, const mla_bf16* w_uv,
                    void* workspace, size_t ws_bytes, mla_bf16* out, float* lse,
                    int32_t* dev_status, void* stream) {
  if (!out) return MLA_ERR_INVALID_ARG;
  return decode_common(dims, q_lat, pool, page_table, seq_lens, batch, nq, max_pages, num_pages, w_uv, 0, 1,
                       workspace, ws_bytes, out, nullptr, lse, dev_status, stream);
}

int mla_decode_attn_partial(const mla_dims* dims, const mla_bf16* q_lat, const mla_bf16* pool,
                            const int32_t* page_table, const int32_t* seq_lens, int32_t batch, int32_t nq,
                            int32_t max_pages, int32_t num_pages, int32_t kv_rank, int32_t kv_ranks,
                            void* workspace, size_t ws_bytes, float* o_lat, float* lse, int32_t* dev_status,
                            void* stream) {
  if (!o_lat || !lse) return MLA_ERR_INVALID_ARG;
  return decode_common(dims, q_lat, pool, page_table, seq_lens, batch, nq, max_pages, num_pages, nullptr, kv_rank,
                       kv_ranks, workspace, ws_bytes, nullptr, o_lat, lse, dev_status, stream);
}

int mla_merge_ranks(const mla_dims* dims, const float* const* o_lat, const float* const* lse, int32_t n_ranks,
                    int32_t n_tokens, const mla_bf16* w_uv, mla_bf16* out, float* lse_out, void* stream) {
  int st = check_dims(dims);
  if (st != MLA_OK) return st;
  if (n_tokens < 0 || n_ranks < 1 || !o_lat || !lse) return MLA_ERR_INVALID_ARG;
  if (n_ranks > mla::kMaxRanks || n_tokens > kMaxMergeTokens) return MLA_ERR_UNSUPPORTED;
  if (n_tokens == 0) return MLA_OK;
  if (!w_uv || !out) return MLA_ERR_INVALID_ARG;
  if (!aligned16(w_uv) || !aligned16(out) || (lse_out && !aligned16(lse_out))) return MLA_ERR_MISALIGNED;
  mla::RankSources src = {};
  src.n = n_ranks;
  for (int r = 0; r < n_ranks; ++r) {
    if (!o_lat[r] || !lse[r]) return MLA_ERR_INVALID_ARG;
    if (!aligned16(o_lat[r]) || !aligned16(lse[r])) return MLA_ERR_MISALIGNED;
    src.o[r] = o_lat[r];
    src.lse[r] = lse[r];
  }
  mla::DecodeArgs a = {};
  a.w_uv = w_uv; a.out = out; a.lse = lse_out;
  a.batch = n_tokens; a.nq = 1; a.n_heads = dims->n_heads; a.d_c = dims->d_c; a.d_rope = dims->d_rope;
  a.v_head = dims->v_head; a.page_size = dims->page_size; a.kv_ranks = 1;
  return cuda_status(mla::launch_merge_ranks(a, src, (cudaStream_t)stream));
}

int mla_out_proj(const mla_dims* dims, const mla_bf16* o, const mla_bf16* w_o, mla_bf16* y,
                 int32_t n_tokens, void* stream) {
  int st = check_dims(dims);
  if (st != MLA_OK) return st;
  if (n_tokens < 0) return MLA_ERR_INVALID_ARG;
  if (n_tokens > kMaxOutProjTokens) return MLA_ERR_UNSUPPORTED;
  if (n_tokens == 0) return MLA_OK;
  if (!o || !w_o || !y) return MLA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(w_o) || !aligned16(y)) return MLA_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_sms(&sms)) != MLA_OK) return st;
  mla::LinearArgs a;
  a.x = o; a.w = w_o; a.y = y;
  a.T = n_tokens; a.K = dims->n_heads * dims->v_head; a.N = dims->d_model;
  a.ksplit = mla::linear_ksplit(a.N, a.K, sms);
  return cuda_status(mla::launch_linear(a, (cudaStream_t)stream));
}

int mla_query_proj(const mla_dims* dims, int32_t q_lora_rank, const mla_bf16* h, const mla_bf16* w_dq,
                   const mla_bf16* w_uq, mla_bf16* c_q, mla_bf16* q, int32_t n_tokens, void* stream) {
  int st = check_dims(dims);
  if (st != MLA_OK) return st;
  if (n_tokens < 0 || q_lora_rank < 1) return MLA_ERR_INVALID_ARG;
  if (n_tokens > kMaxOutProjTokens || q_lora_rank % 8 || q_lora_rank > kMaxQLoraRank) return MLA_ERR_UNSUPPORTED;
  if (n_tokens == 0) return MLA_OK;
  if (!h || !w_dq || !w_uq || !c_q || !q) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_dq) || !aligned16(w_uq) || !aligned16(c_q) || !aligned16(q))
    return MLA_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_sms(&sms)) != MLA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  mla::LinearArgs down;                        // c_Q = W_DQ h
  down.x = h; down.w = w_dq; down.y = c_q;
  down.T = n_tokens; down.K = dims->d_model; down.N = q_lora_rank;
  down.ksplit = mla::linear_ksplit(down.N, down.K, sms);
  if ((st = cuda_status(mla::launch_linear(down, s))) != MLA_OK) return st;
  mla::LinearArgs up;                          // [q_nope || q_rope] per head = W_UQ c_Q
  up.x = c_q; up.w = w_uq; up.y = q;
  up.T = n_tokens; up.K = q_lora_rank; up.N = dims->n_heads * (dims->qk_nope + dims->d_rope);
  up.ksplit = mla::linear_ksplit(up.N, up.K, sms);
  return cuda_status(mla::launch_linear(up, s));
}

int mla_status_read(const int32_t* dev_status, void* stream) {
  if (dev_status == nullptr) return MLA_ERR_INVALID_ARG;
  int32_t v = 0;
  int st = cuda_status(cudaStreamSynchronize((cudaStream_t)stream));
  if (st != MLA_OK) return st;
  if ((st = cuda_status(cudaMemcpy(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost))) != MLA_OK) return st;
  return v;
}

int mla_last_cuda_error(const char** name) {
  const cudaError_t e = g_last_cuda_error;
  if (name != nullptr) *name = cudaGetErrorName(e);
  return (int)e;
}

int mla_status_clear(int32_t* dev_status, void* stream) {
  if (dev_status == nullptr) return MLA_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), (cudaStream_t)stream));
}

const char* mla_status_string(int status) {
  switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: null pointer, bad size or count";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: dimensions not implemented by this build";
    case MLA_ERR_MISALIGNED: return "MLA_ERR_MISALIGNED: pointer not 16-byte aligned";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace too small";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: CUDA runtime error";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT: a bounded device wait ran out";
    case MLA_ERR_RANGE: return "MLA_ERR_RANGE: page id, position or length out of range";
    default: return "unknown mla_status";
  }
}

const char* mla_version(void) { return "mla_b200 0.1.0 sm_100a"; }

}  // extern "C"
