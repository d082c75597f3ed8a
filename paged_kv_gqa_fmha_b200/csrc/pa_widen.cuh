// pa_widen.cuh -- one-time widening of E4M3 K/V pages to bf16 (sm_100a).
//
// The E4M3 KV cache with per-tensor descales ("[Perf][FA4] Warm up dense
// (paged) FA4 attention kernels", vLLM PR #48156, Summary: fp8-descale
// variants of the dense decode and prefill kernels).  A request with two or
// more query blocks reads each of its K/V tiles once per block; widening the
// codes inside the attention kernel would repeat that work for every block
// (about sixteen times per tile on a causal prefill of 1024 tokens).  So the
// pages of such requests are widened once per run into a scratch pool of
// bf16 values, [cap, ps, Hkv, D] like a bf16 pool, and the attention kernel
// reads them as one.  The widening is exact: every E4M3 value (3 mantissa
// bits, exponents 2^-9 .. 2^8) is a bf16 value.  The descales are not applied
// here; they stay in the softmax scale (K) and in 1 / l (V), as for the
// kernels that widen in place.
//
// The scheduler chooses the requests (in request order, while their pages fit
// the pool) and writes wpre[b], the first scratch page of request b; scratch
// page wpre[b] + c holds the request's page c.  This kernel also writes that
// mapping as a dense page table, spt[b * C + c] = wpre[b] + c, for the
// attention kernel.
//
// Grid-stride over (scratch page, K or V): a CTA widens one page part
// (ps * Hkv * D codes) with 16-byte loads and two 16-byte stores per load.
// Bound by HBM: 3 bytes per code (one read, two written).  A page id outside
// [0, num_pages) is reported in the status word and its part is written as
// zeros, as the attention kernels' loaders read such a page.
#pragma once

#include "pa_kernels.cuh"

namespace pa {

struct WidenParams {
  const uint4* k8;            // E4M3 pools [P, ps, Hkv, D] as 16-byte units
  const uint4* v8;
  uint4* k16;                 // scratch pools [cap, ps, Hkv, D] of bf16
  uint4* v16;
  int* spt;                   // [B, C] scratch page table (rows of widened requests)
  const int* page_table;      // [B, tstride]
  const int* wpre;            // [B + 1] first scratch page per request (scheduler)
  const WsHeader* hdr;        // n_wide_pages (scheduler)
  unsigned* status;
  int B, C, tstride, num_pages;
  int part_u4;                // 16-byte units of codes in one page part: ps * Hkv * D / 16
};

constexpr int kWidenThreads = 256;

// Two fp16 (one word) -> two bf16 (one word); exact for the values E4M3 codes
// widen to (fp16 -> fp32 is exact, and 3 mantissa bits fit bf16).
__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t w) {
  float lo, hi;
  asm("{\n\t.reg .b16 a, b;\n\t"
      "mov.b32 {a, b}, %2;\n\t"
      "cvt.f32.f16 %0, a;\n\t"
      "cvt.f32.f16 %1, b;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(w));
  return pack_bf16x2(lo, hi);
}

__global__ void __launch_bounds__(kWidenThreads) pa_widen_kernel(WidenParams p) {
  // the scheduler's outputs (wpre, n_wide_pages) are read below
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int W = p.hdr->n_wide_pages;
  for (int job = blockIdx.x; job < 2 * W; job += gridDim.x) {
    const int gp = job >> 1;
    const bool is_v = (job & 1) != 0;
    // the request owning scratch page gp: the last b with wpre[b] <= gp
    // (requests that were not widened own empty ranges)
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(p.wpre + mid) <= gp) lo = mid; else hi = mid - 1;
    }
    const int b = lo, c = gp - __ldg(p.wpre + b);
    const int page = __ldg(p.page_table + (size_t)b * p.tstride + c);
    const bool bad = page < 0 || (p.num_pages > 0 && page >= p.num_pages);
    if (threadIdx.x == 0) {
      if (bad) atomicOr(p.status, kStatusBadPage);
      if (!is_v) p.spt[(size_t)b * p.C + c] = gp;
    }
    const uint4* src = (is_v ? p.v8 : p.k8) + (size_t)(bad ? 0 : page) * p.part_u4;
    uint4* dst = (is_v ? p.v16 : p.k16) + (size_t)gp * 2 * p.part_u4;
    for (int i = threadIdx.x; i < p.part_u4; i += blockDim.x) {
      const uint4 w = bad ? make_uint4(0u, 0u, 0u, 0u) : __ldg(src + i);
      const uint32_t in[4] = {w.x, w.y, w.z, w.w};
      uint32_t o[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t f0, f1;
        e4m3x4_to_f16x4(in[e], f0, f1);
        o[2 * e] = f16x2_to_bf16x2(f0);
        o[2 * e + 1] = f16x2_to_bf16x2(f1);
      }
      dst[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace pa
