// Linear maps of the decode step's few tokens: y[t] = W x[t] for T tokens, with
// W [N, K] bf16 in nn.Linear orientation.  Two calls use it:
//   mla_query_proj  c_Q = W_DQ h, then [q_nope || q_rope] = W_UQ c_Q per head
//                   ("DeepSeek MLA Architecture: How It Cuts KV Cache by 93%",
//                   sec. 3: q_lora_rank 1536; "MHA vs MLA KV cache comparison",
//                   "Note on Actual Implementation": the query side is down- then
//                   up-projected)
//   mla_out_proj    y = W_O concat_h(o_h) ("Deep-Dive: Multi-Head Latent Attention
//                   (MLA) and Low-Rank KV Cache Compression in DeepSeek-V3", sec. 3:
//                   out_proj over the head-major concatenation; "mla-from-scratch"
//                   README, "Absorption, and why RoPE breaks it": W_UV is applied
//                   once after attending, next to W_O)
//
// With T = 16 (the V3-shaped step) each is a stream of W (22 MB W_DQ, 75 MB W_UQ,
// 235 MB W_O) against a small activation block that stays in L2: HBM-bound, 2 T
// flops per weight element.  Tensor cores are used through warp-level mma.sync
// tiles because T is far below the 128-row minimum of a tcgen05 tile; what sets
// the speed is keeping enough weight bytes in flight on every SM.
//
// CTA = 4 warps on one 16-row tile of W (16 outputs) and 8 * NT tokens.  The
// reduction index is cut into 32-wide slices; each thread loads its 16-byte pieces
// of two weight rows (evict-first) and of NT token rows (L2) per slice (fragment
// convention of mma_frag.cuh), several slices ahead, and the warps take the
// slices round-robin.  When W has too few rows to give every SM work (W_DQ: 96
// tiles), the slices are also split over a cluster of `ksplit` CTAs, whose partial
// tiles are summed in the cluster leader's shared memory.  One bf16 rounding per
// output.
#include "../../include/mla.h"
#include "common.cuh"
#include "decode.h"
#include "mma_frag.cuh"
#include "sm100.cuh"

namespace mla {

namespace {

using sm100::cluster_arrive_relaxed;
using sm100::cluster_sync;
using sm100::cluster_wait;
using sm100::mapa;
using sm100::smem_u32;

constexpr int kLinWarps = 4;
constexpr int kLinThreads = kLinWarps * 32;
constexpr int kLinRows = 16;       // outputs (rows of W) per CTA
constexpr int kLinMaxSplit = 8;    // portable cluster size

template <int NT>
struct LinUnroll {
  static constexpr int value = NT <= 2 ? 4 : 2;  // slices in flight per warp (register budget)
};

// NT: n8 token tiles per CTA (8 * NT tokens); SPLIT: the reduction is split over
// a cluster of a.ksplit CTAs.  Only the split form holds the leader's buffer for
// the partial tiles: the plain form keeps its shared memory small, which leaves
// the SM a large L1 for the token rows its CTAs read in step.
template <int NT, bool SPLIT>
__global__ void __launch_bounds__(kLinThreads, 4) token_linear_kernel(const LinearArgs a) {
  constexpr int U = LinUnroll<NT>::value;
  constexpr int kTile = 32 * NT * 4;                   // fp32 values of a CTA's output tile
  __shared__ float red[kLinWarps][32][NT * 4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int ks = SPLIT ? a.ksplit : 1;
  const int kr = SPLIT ? blockIdx.x % ks : 0;          // rank in the cluster (clusters run along x)
  const int r0 = (blockIdx.x / ks) * kLinRows;
  const int t0 = blockIdx.y * 8 * NT;
  const int K = a.K;
  const int nslices = (K + 31) / 32;
  const int per = (nslices + ks - 1) / ks;
  const int s_lo = kr * per, s_hi = min(nslices, s_lo + per);
  // rows g and g + 8 of the tile; rows past N read row 0 and are masked
  const bool ra_ok = r0 + g < a.N, rb_ok = r0 + g + 8 < a.N;
  const uint16_t* wa = a.w + (size_t)(ra_ok ? r0 + g : 0) * K + 8 * q;
  const uint16_t* wb = a.w + (size_t)(rb_ok ? r0 + g + 8 : 0) * K + 8 * q;
  const uint16_t* xr[NT];
  bool x_ok[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int tok = t0 + 8 * j + g;
    x_ok[j] = tok < a.T;
    xr[j] = a.x + (size_t)(x_ok[j] ? tok : 0) * K + 8 * q;
  }
  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

  const uint4 zero = make_uint4(0, 0, 0, 0);
  uint4 a0[U], a1[U];
  // the weight pieces of the batch of slices that starts at s0
  auto load_w = [&](int s0) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int s = s0 + u * kLinWarps;
      const int k = 32 * s;
      // K is a multiple of 8: a thread's 8-element piece is wholly inside or outside
      const bool k_ok = s < s_hi && k + 8 * q < K;
      a0[u] = (k_ok && ra_ok) ? ldg_stream(wa + k) : zero;
      a1[u] = (k_ok && rb_ok) ? ldg_stream(wb + k) : zero;
    }
  };
  // The first batch of weights is in flight before the dependency wait, while the
  // preceding kernel on the stream finishes (the kernel enqueued just before the
  // call must not write W; every kernel here allows its dependents only after its
  // own wait, so everything earlier on the stream has completed).
  load_w(s_lo + warp);
  if (SPLIT) cluster_arrive_relaxed();  // paired with the wait before the first remote store
  grid_dependency_wait();  // x is written by the preceding kernel
  allow_dependent_launch();

  for (int s0 = s_lo + warp; s0 < s_hi; s0 += kLinWarps * U) {
    uint4 b[U][NT];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int s = s0 + u * kLinWarps;
      const int k = 32 * s;
      const bool k_ok = s < s_hi && k + 8 * q < K;
#pragma unroll
      for (int j = 0; j < NT; ++j)
        b[u][j] = (k_ok && x_ok[j]) ? __ldg(reinterpret_cast<const uint4*>(xr[j] + k)) : zero;
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int j = 0; j < NT; ++j) mma_k32(acc[j], a0[u], a1[u], b[u][j]);
    if (s0 + kLinWarps * U < s_hi) load_w(s0 + kLinWarps * U);
  }

#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) red[warp][lane][4 * j + c] = acc[j][c];
  __syncthreads();
  // element i of the tile: lane ln = i % 32 of the fragment, e = i / 32; token
  // tile j = e / 4, c = e % 4 gives row g (+8 for c >= 2) and token 2q (+1 for odd c)
  auto warp_sum = [&](int i) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kLinWarps; ++w) v += red[w][i % 32][i / 32];
    return v;
  };
  auto store = [&](int i, float v) {
    const int e = i / 32, ln = i % 32;
    const int row = r0 + (ln >> 2) + ((e & 2) ? 8 : 0);
    const int tok = t0 + 8 * (e >> 2) + 2 * (ln & 3) + (e & 1);
    if (row < a.N && tok < a.T) a.y[(size_t)tok * a.N + row] = f32_to_bf16(v);
  };
  if constexpr (SPLIT) {
    __shared__ float split_part[kLinMaxSplit][kTile];  // cluster leader: the split CTAs' tiles
    // partial tile -> the leader's slot kr (distributed shared memory), once
    // every CTA of the cluster is known to have started
    cluster_wait();
    const uint32_t dst = mapa(smem_u32(&split_part[kr][0]), 0);
    for (int i = threadIdx.x; i < kTile; i += kLinThreads)
      asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(dst + 4 * i), "f"(warp_sum(i)) : "memory");
    cluster_sync();  // every split CTA's tile is in the leader's shared memory
    if (kr != 0) return;
    for (int i = threadIdx.x; i < kTile; i += kLinThreads) {
      float v = 0.f;
      for (int r = 0; r < ks; ++r) v += split_part[r][i];
      store(i, v);
    }
  } else {
    for (int i = threadIdx.x; i < kTile; i += kLinThreads) store(i, warp_sum(i));
  }
}

template <int NT, bool SPLIT>
cudaError_t launch_nt(const LinearArgs& a, cudaStream_t stream) {
  cudaLaunchAttribute attr[2] = {pdl_attribute(), {}};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.N + kLinRows - 1) / kLinRows * a.ksplit, (a.T + 8 * NT - 1) / (8 * NT), 1);
  cfg.blockDim = dim3(kLinThreads, 1, 1);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (SPLIT) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = a.ksplit;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, token_linear_kernel<NT, SPLIT>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int NT>
cudaError_t launch_nt(const LinearArgs& a, cudaStream_t stream) {
  return a.ksplit > 1 ? launch_nt<NT, true>(a, stream) : launch_nt<NT, false>(a, stream);
}

}  // namespace

int linear_ksplit(int N, int K, int sms) {
  // enough CTAs for two per SM when W has few rows, while each split CTA keeps
  // at least 16 slices (512 columns) of every row
  const int tiles = (N + kLinRows - 1) / kLinRows;
  int ks = 1;
  while (ks < kLinMaxSplit && tiles * ks < 2 * sms && (K / 32) / (2 * ks) >= 16) ks *= 2;
  return ks;
}

cudaError_t launch_linear(const LinearArgs& a, cudaStream_t stream) {
  if (a.ksplit < 1 || a.ksplit > kLinMaxSplit) return cudaErrorInvalidValue;
  if (a.T <= 8) return launch_nt<1>(a, stream);
  if (a.T <= 16) return launch_nt<2>(a, stream);
  return launch_nt<4>(a, stream);  // 32 tokens per CTA row of the grid
}

}  // namespace mla
