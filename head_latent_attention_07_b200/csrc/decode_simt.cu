// Split-KV latent attention on CUDA cores (any supported shape).
//
// One CTA = (worker w, group of kRows query rows).  A query row is one
// (query token i, head h) pair of a sequence; the rows of a sequence are its
// nq*H rows in q_lat order.  The worker walks its chunk of pages (see plan.cuh);
// each page [page_size, d_c + d_rope] is staged once in shared memory and used
// for both products:
//   s[r][n]  = scale * q_lat[r] . page[n]          (content + positional term)
//   online softmax over the pages of the piece (running max m, sum l, in log2 units)
//   O[r][:] += p[r][n] * page[n][0:d_c]            (values read in latent space)
// and at the end of each piece writes O/l and lse = ln(sum exp s) to the workspace.
#include "common.cuh"
#include "plan.cuh"
#include "decode.h"

namespace mla {

namespace {

constexpr int kThreads = 256;
constexpr int kRows = 16;  // query rows per CTA

struct SimtSmem {
  PlanSmem plan;
  float m[kRows];
  float l[kRows];
  float alpha[kRows];
};

__global__ void __launch_bounds__(kThreads)
decode_split_simt_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem* sm = reinterpret_cast<SimtSmem*>(smem_raw);
  const int R = a.d_c + a.d_rope;
  const int rows_total = a.nq * a.n_heads;
  float* q_s = reinterpret_cast<float*>(smem_raw + ((sizeof(SimtSmem) + 15) & ~size_t(15)));  // [kRows][R]
  uint16_t* page_s = reinterpret_cast<uint16_t*>(q_s + kRows * R);                           // [P][R]
  float* s_s = reinterpret_cast<float*>(page_s + a.page_size * R);                            // [kRows][P]

  grid_dependency_wait();
  allow_dependent_launch();   // only after the wait: the combine reads seq_lens and W_UV, written before this kernel's wait returned
  build_plan(&sm->plan, a.seq_lens, a.batch, a.nq, a.max_pages, a.page_size, a.G, a.piece_cost, a.dev_status,
             a.kv_rank, a.kv_ranks);
  const int w = blockIdx.x;
  const int row0 = blockIdx.y * kRows;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = a.page_size;
  const float sl2 = a.scale * 1.4426950408889634f;  // scale * log2(e)
  const int rv = R / 8;                             // 16-byte vectors per cache row
  // value-phase ownership: one 8-column vector, 4 rows
  const int cv = tid % 64;
  const int rq = (tid / 64) * 4;
  const bool own_cols = cv < a.d_c / 8;

  PieceIter it(&sm->plan, a.batch, w);
  Piece pc;
  while (it.next(&pc)) {
    const int b = pc.b;
    const int piece = pc.id;
    const int len = a.seq_lens[b];

    // query rows of this sequence -> fp32 shared memory
    const uint16_t* qb = a.q_lat + (size_t)b * rows_total * R;
    for (int idx = tid; idx < kRows * rv; idx += kThreads) {
      int j = idx / rv, v = idx % rv;
      float fv[8];
      if (row0 + j < rows_total) {
        uint4 u = *reinterpret_cast<const uint4*>(qb + (size_t)(row0 + j) * R + v * 8);
        unpack8(u, fv);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) fv[k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) q_s[j * R + v * 8 + k] = fv[k];
    }
    if (tid < kRows) { sm->m[tid] = -INFINITY; sm->l[tid] = 0.f; }
    float acc[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[r][k] = 0.f;
    __syncthreads();

    for (int pg = pc.pg_begin; pg < pc.pg_end; ++pg) {   // absolute page indices of the sequence
      const int page_id = a.page_table[(size_t)b * a.max_pages + pg];
      if (page_id < 0 || page_id >= a.num_pages) {  // uniform across the CTA
        if (tid == 0) record_status(a.dev_status, MLA_ERR_RANGE);
        continue;
      }
      const int base = pg * P;
      const int nvalid = min(P, len - base);
      const uint16_t* src = a.pool + (size_t)page_id * P * R;
      for (int idx = tid; idx < P * rv; idx += kThreads) {
        int n = idx / rv;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (n < nvalid) u = ldg_stream(src + (size_t)idx * 8);  // slots past the length read as 0
        reinterpret_cast<uint4*>(page_s)[idx] = u;
      }
      __syncthreads();

      // scores: warp handles tokens warp, warp+8, ...; lanes split the row
      for (int n = warp; n < P; n += kThreads / 32) {
        float part[kRows];
#pragma unroll
        for (int j = 0; j < kRows; ++j) part[j] = 0.f;
        for (int v = lane; v < rv; v += 32) {
          float kv[8];
          unpack8(reinterpret_cast<const uint4*>(page_s + n * R)[v], kv);
#pragma unroll
          for (int j = 0; j < kRows; ++j) {
            const float4 q0 = *reinterpret_cast<const float4*>(q_s + j * R + v * 8);
            const float4 q1 = *reinterpret_cast<const float4*>(q_s + j * R + v * 8 + 4);
            part[j] += q0.x * kv[0] + q0.y * kv[1] + q0.z * kv[2] + q0.w * kv[3] +
                       q1.x * kv[4] + q1.y * kv[5] + q1.z * kv[6] + q1.w * kv[7];
          }
        }
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          float t = warp_sum(part[j]);
          if (lane == j) {
            const int row = row0 + j;
            const int qi = row / a.n_heads;                 // query token of this row
            const bool vis = row < rows_total && base + n <= len - a.nq + qi;
            s_s[j * P + n] = vis ? t * sl2 : -INFINITY;
          }
        }
      }
      __syncthreads();

      // online softmax: two rows per warp
      for (int j = warp; j < kRows; j += kThreads / 32) {
        float mx = -INFINITY;
        for (int n = lane; n < P; n += 32) mx = fmaxf(mx, s_s[j * P + n]);
        mx = warp_max(mx);
        const float m_old = sm->m[j];
        const float m_new = fmaxf(m_old, mx);
        float sum = 0.f;
        for (int n = lane; n < P; n += 32) {
          float s = s_s[j * P + n];
          float p = (s == -INFINITY) ? 0.f : exp2f(s - m_new);
          s_s[j * P + n] = p;
          sum += p;
        }
        sum = warp_sum(sum);
        __syncwarp();
        if (lane == 0) {
          const float alpha = (m_old == -INFINITY) ? 0.f : exp2f(m_old - m_new);
          sm->alpha[j] = alpha;
          sm->l[j] = sm->l[j] * alpha + sum;
          sm->m[j] = m_new;
        }
      }
      __syncthreads();

      // values: O[r][cols] = alpha * O + sum_n p[r][n] * c_n[cols]
      if (own_cols) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float al = sm->alpha[rq + r];
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[r][k] *= al;
        }
        for (int n = 0; n < P; ++n) {
          float cvv[8];
          unpack8(reinterpret_cast<const uint4*>(page_s + n * R)[cv], cvv);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float p = s_s[(rq + r) * P + n];
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[r][k] += p * cvv[k];
          }
        }
      }
      __syncthreads();  // page_s / s_s are rewritten by the next page
    }

    // piece result: O / l and lse (natural log); rows that saw no key: 0, -inf
    float* po = a.part_o + (size_t)piece * rows_total * a.d_c;
    float* pl = a.part_lse + (size_t)piece * rows_total;
    if (own_cols) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = row0 + rq + r;
        if (row >= rows_total) continue;
        const float l = sm->l[rq + r];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float4* dst = reinterpret_cast<float4*>(po + (size_t)row * a.d_c + cv * 8);
        dst[0] = make_float4(acc[r][0] * inv, acc[r][1] * inv, acc[r][2] * inv, acc[r][3] * inv);
        dst[1] = make_float4(acc[r][4] * inv, acc[r][5] * inv, acc[r][6] * inv, acc[r][7] * inv);
      }
    }
    if (tid < kRows && row0 + tid < rows_total) {
      const float l = sm->l[tid];
      pl[row0 + tid] = l > 0.f ? (sm->m[tid] + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
    __syncthreads();
  }
}

}  // namespace

size_t decode_simt_smem_bytes(int d_c, int d_rope, int page_size) {
  const int R = d_c + d_rope;
  return ((sizeof(SimtSmem) + 15) & ~size_t(15)) + (size_t)kRows * R * 4 + (size_t)page_size * R * 2 +
         (size_t)kRows * page_size * 4;
}

int decode_simt_row_groups(int rows_total) { return (rows_total + kRows - 1) / kRows; }

cudaError_t launch_decode_split_simt(const DecodeArgs& a, cudaStream_t stream) {
  const size_t smem = decode_simt_smem_bytes(a.d_c, a.d_rope, a.page_size);
  cudaError_t e = cudaFuncSetAttribute(decode_split_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.G, decode_simt_row_groups(a.nq * a.n_heads));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_split_simt_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mla
