// mla_append_latent and mla_absorb_q kernels.
//
// append:  [c_t || k^_t] = w_dkv h_t (c_t = W_DKV h_t, k^_t = W_KR h_t), k_t^R =
//          RoPE(k^_t, pos_t); the bf16 row goes to its paged cache slot.
// absorb:  q_lat[t][h] = [W_UK,h^T q_nope || RoPE(q_rope, pos_t)].
// Both are weight-read bound (w_dkv 8.3 MB, W_UK 16.8 MB at DeepSeek-V3 shape):
// each CTA streams its slice of the weights once and applies it to a block of
// up to 16 tokens held on chip.
#include "common.cuh"
#include "decode.h"

namespace mla {

namespace {

constexpr int kTokBlk = 16;

// ------------------------------------------------------------------ append
constexpr int kAppRows = 4;     // output rows (of d_c + d_rope) per CTA, one per warp
constexpr int kAppK = 1024;     // hidden-state columns staged per step

__global__ void __launch_bounds__(kAppRows * 32)
append_latent_kernel(AppendArgs a) {
  __shared__ __align__(16) uint16_t h_s[kTokBlk * kAppK];
  __shared__ float vals[kAppRows][kTokBlk];
  const int R = a.d_c + a.d_rope;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r0 = blockIdx.x * kAppRows;
  const int t0 = blockIdx.y * kTokBlk;
  const int r = r0 + warp;
  float acc[kTokBlk];
#pragma unroll
  for (int j = 0; j < kTokBlk; ++j) acc[j] = 0.f;

  for (int k0 = 0; k0 < a.d_model; k0 += kAppK) {
    for (int idx = threadIdx.x; idx < kTokBlk * (kAppK / 8); idx += blockDim.x) {
      const int j = idx / (kAppK / 8), v = idx % (kAppK / 8);
      const int col = k0 + v * 8;
      uint4 u = make_uint4(0, 0, 0, 0);
      if (t0 + j < a.n_tokens && col < a.d_model)
        u = *reinterpret_cast<const uint4*>(a.h + (size_t)(t0 + j) * a.d_model + col);
      reinterpret_cast<uint4*>(h_s)[idx] = u;
    }
    __syncthreads();
    if (r < R) {
      const uint16_t* wrow = a.w_dkv + (size_t)r * a.d_model + k0;
      const int nv = min(kAppK, a.d_model - k0) / 8;
      for (int v = lane; v < nv; v += 32) {
        float wv[8];
        unpack8(ldg_stream(wrow + v * 8), wv);
#pragma unroll
        for (int j = 0; j < kTokBlk; ++j) {
          float hv[8];
          unpack8(reinterpret_cast<const uint4*>(h_s + j * kAppK)[v], hv);
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[j] += wv[k] * hv[k];
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < kTokBlk; ++j) {
    const float s = warp_sum(acc[j]);
    if (lane == j) vals[warp][j] = s;
  }
  __syncthreads();

  // store: thread (row rr, token j); RoPE rows pair up inside the CTA
  // (r0 and d_c are multiples of kAppRows, hence even)
  for (int idx = threadIdx.x; idx < kAppRows * kTokBlk; idx += blockDim.x) {
    const int rr = idx / kTokBlk, j = idx % kTokBlk;
    const int row = r0 + rr, t = t0 + j;
    if (row >= R || t >= a.n_tokens) continue;
    const int seq = a.seq_idx[t], p = a.pos[t];
    if (seq < 0 || seq >= a.batch || p < 0 || p >= a.max_pages * a.page_size) {
      record_status(a.dev_status, MLA_ERR_RANGE);
      continue;
    }
    const int page = a.page_table[(size_t)seq * a.max_pages + p / a.page_size];
    if (page < 0 || page >= a.num_pages) {
      record_status(a.dev_status, MLA_ERR_RANGE);
      continue;
    }
    float val = vals[rr][j];
    if (row >= a.d_c) {
      const int q = row - a.d_c;          // channel within the RoPE key
      float c, s;
      rope_cos_sin(p, q >> 1, a.d_rope, a.theta, &c, &s);
      const float x0 = vals[rr & ~1][j], x1 = vals[rr | 1][j];
      val = (q & 1) ? x0 * s + x1 * c : x0 * c - x1 * s;
    }
    a.pool[((size_t)page * a.page_size + p % a.page_size) * R + row] = f32_to_bf16(val);
  }
}

// ------------------------------------------------------------------ absorb
constexpr int kAbsThreads = 256;

__global__ void __launch_bounds__(kAbsThreads)
absorb_q_kernel(AbsorbArgs a) {
  extern __shared__ __align__(16) float qn[];   // [kTokBlk][qk_nope]
  const int h = blockIdx.x;
  const int t0 = blockIdx.y * kTokBlk;
  const int dq = a.qk_nope + a.d_rope;
  const int R = a.d_c + a.d_rope;
  for (int idx = threadIdx.x; idx < kTokBlk * a.qk_nope; idx += blockDim.x) {
    const int j = idx / a.qk_nope, i = idx % a.qk_nope;
    const int t = t0 + j;
    qn[idx] = t < a.n_tokens ? bf16_to_f32(a.q[((size_t)t * a.n_heads + h) * dq + i]) : 0.f;
  }
  __syncthreads();
  const uint16_t* wh = a.w_uk + (size_t)h * a.qk_nope * a.d_c;
  // content part: thread owns column pairs (j, j+1)
  for (int j = 2 * threadIdx.x; j < a.d_c; j += 2 * blockDim.x) {
    float acc0[kTokBlk], acc1[kTokBlk];
#pragma unroll
    for (int k = 0; k < kTokBlk; ++k) { acc0[k] = 0.f; acc1[k] = 0.f; }
    for (int i = 0; i < a.qk_nope; ++i) {
      const uint32_t w2 = *reinterpret_cast<const uint32_t*>(wh + (size_t)i * a.d_c + j);
      const float w0 = bf16_lo(w2), w1 = bf16_hi(w2);
#pragma unroll
      for (int k = 0; k < kTokBlk; ++k) {
        const float qv = qn[k * a.qk_nope + i];
        acc0[k] += w0 * qv;
        acc1[k] += w1 * qv;
      }
    }
#pragma unroll
    for (int k = 0; k < kTokBlk; ++k) {
      const int t = t0 + k;
      if (t < a.n_tokens)
        *reinterpret_cast<uint32_t*>(a.q_lat + ((size_t)t * a.n_heads + h) * R + j) =
            pack_bf16x2(acc0[k], acc1[k]);
    }
  }
  // positional part: RoPE(q_rope, pos)
  const int npair = a.d_rope / 2;
  for (int idx = threadIdx.x; idx < kTokBlk * npair; idx += blockDim.x) {
    const int k = idx / npair, i = idx % npair;
    const int t = t0 + k;
    if (t >= a.n_tokens) continue;
    const uint16_t* src = a.q + ((size_t)t * a.n_heads + h) * dq + a.qk_nope + 2 * i;
    const float x0 = bf16_to_f32(src[0]), x1 = bf16_to_f32(src[1]);
    float c, s;
    rope_cos_sin(a.pos[t], i, a.d_rope, a.theta, &c, &s);
    *reinterpret_cast<uint32_t*>(a.q_lat + ((size_t)t * a.n_heads + h) * R + a.d_c + 2 * i) =
        pack_bf16x2(x0 * c - x1 * s, x0 * s + x1 * c);
  }
}

}  // namespace

cudaError_t launch_append_latent(const AppendArgs& a, cudaStream_t stream) {
  const int R = a.d_c + a.d_rope;
  dim3 grid((R + kAppRows - 1) / kAppRows, (a.n_tokens + kTokBlk - 1) / kTokBlk);
  append_latent_kernel<<<grid, kAppRows * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_absorb_q(const AbsorbArgs& a, cudaStream_t stream) {
  const size_t smem = (size_t)kTokBlk * a.qk_nope * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(absorb_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(a.n_heads, (a.n_tokens + kTokBlk - 1) / kTokBlk);
  absorb_q_kernel<<<grid, kAbsThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
