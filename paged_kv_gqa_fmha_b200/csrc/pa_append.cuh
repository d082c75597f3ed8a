// pa_append.cuh -- paged KV append (sm_100a).
//
// The step before attention in serving: this step's new K and V rows are
// written into the page pool ("integrate PrimTS FMHA kernels", TensorRT-LLM
// PR #17399, section "Planning, preprocessing, and workspace ownership": the
// KV-cache append of the fused preprocessing; the slot follows section
// "Unified page-table metadata").  New token i of request b (packed row
// cu[b] + i of k_new / v_new) is KV position j = kv_b - q_b + i and goes to
// page page_table[b][j / ps], slot j % ps, all KV heads at once: the row of a
// slot, [Hkv, D], is contiguous in the [P, ps, Hkv, D] pool.
//
// One warp per new token: find the request by binary search over cu_q_lens,
// then copy the K row and the V row with 16-byte loads and stores (lanes over
// the row, so every warp access is contiguous).  Bound by HBM: 2 * 2 * Hkv * D
// * 2 bytes per token (read and write, K and V).
//
// What cannot be placed is skipped and reported in the status word: a token
// on a page id outside [0, num_pages) (that token), q_b > kv_b or
// kv_b > C * ps (the request), malformed cu_q_lens (nothing is written; every
// CTA checks it before copying anything).
#pragma once

#include "pa_kernels.cuh"

namespace pa {

struct AppendParams {
  const uint4* k_new;         // bf16 [T, Hkv, D] as 16-byte units
  const uint4* v_new;
  uint4* k_pool;              // bf16 [P, ps, Hkv, D]
  uint4* v_pool;
  const int* page_table;      // [B, C]
  const int* seq_lens;        // [B]
  const int* cu_q_lens;       // [B+1] or nullptr (one token per request)
  unsigned* status;
  int B, C, ps, num_pages;
  int tstride;                // page-table row stride (>= C)
  int row_u4;                 // 16-byte units of one token's K (or V) row: Hkv * D / 8
};

constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads) pa_append_kernel(AppendParams p) {
  __shared__ int bad_cu;
  // cu_q_lens must start at 0 and never decrease; otherwise write nothing
  if (threadIdx.x == 0) bad_cu = 0;
  __syncthreads();
  if (p.cu_q_lens) {
    // (cu[B] past B * C * ps also implies some q_b > C * ps >= kv_b)
    int bad = (threadIdx.x == 0 && (p.cu_q_lens[0] != 0 ||
                                     (long)p.cu_q_lens[p.B] > (long)p.B * p.C * p.ps)) ? 1 : 0;
    for (int b = threadIdx.x; b < p.B; b += blockDim.x)
      if (p.cu_q_lens[b + 1] < p.cu_q_lens[b]) bad = 1;
    if (bad) atomicOr(&bad_cu, 1);
  }
  __syncthreads();
  if (bad_cu) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, kStatusBadCuQ);
    return;
  }
  const int lane = threadIdx.x & 31;
  const long n_warps = (long)gridDim.x * (blockDim.x >> 5);
  const long T = p.cu_q_lens ? p.cu_q_lens[p.B] : p.B;
  for (long t = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += n_warps) {
    int b = (int)t;
    if (p.cu_q_lens) {
      // largest b with cu[b] <= t (cu is nondecreasing and cu[B] = T > t)
      int lo = 0, hi = p.B;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.cu_q_lens[mid] <= t) lo = mid;
        else hi = mid;
      }
      b = lo;
    }
    const long t0 = p.cu_q_lens ? p.cu_q_lens[b] : b;
    const int qb = p.cu_q_lens ? p.cu_q_lens[b + 1] - p.cu_q_lens[b] : 1;
    const int kv = p.seq_lens[b];
    const int i = (int)(t - t0);
    if (qb > kv) {
      if (lane == 0 && i == 0) atomicOr(p.status, kStatusQgtKv);
      continue;
    }
    if ((long)kv > (long)p.C * p.ps) {
      if (lane == 0 && i == 0) atomicOr(p.status, kStatusKvGtCap);
      continue;
    }
    const int j = kv - qb + i;
    const int page = __ldg(p.page_table + (size_t)b * p.tstride + j / p.ps);
    if (page < 0 || (p.num_pages > 0 && page >= p.num_pages)) {
      if (lane == 0) atomicOr(p.status, kStatusBadPage);
      continue;
    }
    const size_t src = (size_t)t * p.row_u4;
    const size_t dst = ((size_t)page * p.ps + j % p.ps) * p.row_u4;
    // all loads of a chunk before its stores: 8 x 16 bytes in flight per lane
    for (int u0 = 0; u0 < p.row_u4; u0 += 4 * 32) {
      uint4 kx[4], vx[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int u = u0 + k * 32 + lane;
        if (u < p.row_u4) {
          kx[k] = __ldg(p.k_new + src + u);
          vx[k] = __ldg(p.v_new + src + u);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int u = u0 + k * 32 + lane;
        if (u < p.row_u4) {
          p.k_pool[dst + u] = kx[k];
          p.v_pool[dst + u] = vx[k];
        }
      }
    }
  }
}

}  // namespace pa
