// Combine of the split-KV partials, then the W_UV up-projection.
//
// For query row (token t, head h) with pieces s of its sequence:
//   LSE   = ln sum_s exp(lse_s)
//   o_lat = sum_s exp(lse_s - LSE) * O_s          (O_s already normalised per piece)
//   out[t][h][v] = sum_c W_UV[h][v][c] * o_lat[c]  (values up-projected once, after
//                                                   attending over latents)
// One CTA = one head and up to kTok query tokens, so W_UV,h is streamed once per
// group of kTok tokens and reused from registers across them.
#include "common.cuh"
#include "plan.cuh"
#include "decode.h"

namespace mla {

namespace {

constexpr int kThreads = 256;
constexpr int kTok = 16;

__global__ void __launch_bounds__(kThreads)
decode_combine_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  PlanSmem* ps = reinterpret_cast<PlanSmem*>(smem_raw);
  float* olat = reinterpret_cast<float*>(smem_raw + ((sizeof(PlanSmem) + 15) & ~size_t(15)));  // [kTok][d_c]

  build_plan(ps, a.seq_lens, a.batch, a.nq, a.max_pages, a.page_size, a.G, nullptr);
  const int h = blockIdx.x;
  const int t0 = blockIdx.y * kTok;
  const int T = a.batch * a.nq;
  const int rows_total = a.nq * a.n_heads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // 1. merge: one warp per token
  for (int j = warp; j < kTok; j += kThreads / 32) {
    const int t = t0 + j;
    float* dst = olat + j * a.d_c;
    if (t >= T) {
      for (int c = lane; c < a.d_c; c += 32) dst[c] = 0.f;
      continue;
    }
    const int b = t / a.nq, i = t % a.nq;
    const int row = i * a.n_heads + h;
    const int pb = ps->piece_begin[b], np = ps->piece_begin[b + 1] - pb;
    float mx = -INFINITY;
    for (int s = lane; s < np; s += 32) mx = fmaxf(mx, a.part_lse[(size_t)(pb + s) * rows_total + row]);
    mx = warp_max(mx);
    float tot = 0.f;
    for (int s = lane; s < np; s += 32) {
      const float l = a.part_lse[(size_t)(pb + s) * rows_total + row];
      tot += (l == -INFINITY) ? 0.f : expf(l - mx);
    }
    tot = warp_sum(tot);
    const bool empty = (mx == -INFINITY);
    const float lse_all = empty ? -INFINITY : mx + logf(tot);
    for (int c = lane * 4; c < a.d_c; c += 128) {
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (!empty) {
        for (int s = 0; s < np; ++s) {
          const float l = a.part_lse[(size_t)(pb + s) * rows_total + row];
          if (l == -INFINITY) continue;
          const float wgt = expf(l - lse_all);
          const float4 v = *reinterpret_cast<const float4*>(
              a.part_o + ((size_t)(pb + s) * rows_total + row) * a.d_c + c);
          o.x += wgt * v.x; o.y += wgt * v.y; o.z += wgt * v.z; o.w += wgt * v.w;
        }
      }
      *reinterpret_cast<float4*>(dst + c) = o;
    }
    if (lane == 0 && a.lse != nullptr) a.lse[(size_t)t * a.n_heads + h] = lse_all;
  }
  __syncthreads();

  // 2. out[t][h][v] = W_UV,h[v] . o_lat[t]: warp per value row, lanes split d_c
  const int cvec = a.d_c / 8;
  const uint16_t* wh = a.w_uv + (size_t)h * a.v_head * a.d_c;
  for (int v = warp; v < a.v_head; v += kThreads / 32) {
    float part[kTok];
#pragma unroll
    for (int j = 0; j < kTok; ++j) part[j] = 0.f;
    for (int k = lane; k < cvec; k += 32) {
      float wv[8];
      unpack8(ldg_stream(wh + (size_t)v * a.d_c + k * 8), wv);
#pragma unroll
      for (int j = 0; j < kTok; ++j) {
        const float4 o0 = *reinterpret_cast<const float4*>(olat + j * a.d_c + k * 8);
        const float4 o1 = *reinterpret_cast<const float4*>(olat + j * a.d_c + k * 8 + 4);
        part[j] += wv[0] * o0.x + wv[1] * o0.y + wv[2] * o0.z + wv[3] * o0.w +
                   wv[4] * o1.x + wv[5] * o1.y + wv[6] * o1.z + wv[7] * o1.w;
      }
    }
#pragma unroll
    for (int j = 0; j < kTok; ++j) {
      const float sum = warp_sum(part[j]);
      const int t = t0 + j;
      if (lane == j && t < T) a.out[((size_t)t * a.n_heads + h) * a.v_head + v] = f32_to_bf16(sum);
    }
  }
}

}  // namespace

cudaError_t launch_decode_combine(const DecodeArgs& a, cudaStream_t stream) {
  const size_t smem = ((sizeof(PlanSmem) + 15) & ~size_t(15)) + (size_t)kTok * a.d_c * 4;
  cudaError_t e = cudaFuncSetAttribute(decode_combine_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int T = a.batch * a.nq;
  dim3 grid(a.n_heads, (T + kTok - 1) / kTok);
  decode_combine_kernel<<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
