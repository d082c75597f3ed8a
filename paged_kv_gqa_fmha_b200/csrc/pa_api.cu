// pa_api.cu -- the C ABI declared in include/pa.h.
//
// Host side only: argument validation, plan / workspace ownership, TMA tensor
// maps for the q tensor and the two page pools, and the three launches.  No
// host <-> device synchronisation happens in pa_run, so it can be captured in
// a CUDA graph (decode is run as FULL CUDA graphs in the FA4 warm-up PR, vLLM
// #48156; PrimTS tests generation CUDA-graph replay, TensorRT-LLM #17399).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/pa.h"
#include "pa_kernels.cuh"
#include "pa_prefill.cuh"
#include "pa_decode.cuh"
#include "pa_append.cuh"
#include "pa_widen.cuh"

namespace {

thread_local char g_err[512] = "";

void set_err(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

// What the scheduler writes and the attention and merge kernels of the same
// run read.  Two sets, used by alternate runs: a run's scheduler may start
// (as a programmatic dependent) while the previous run's kernels still read
// the other set; it waits for them before it exits.
struct SchedBufs {
  pa::WsHeader* hdr;          // n_items, n_split_reqs, n_items2 (status is in set 0)
  int4* req_info;
  int4* req_aux;
  int* unit_off;
  int* split_list;
  pa::PackedItem* items;
  int* unit_off2;
  pa::PackedItem* items2;
  int* split_cnt;             // [B * Hkv] fused-merge counters (plans with splits)
  int* wpre;                  // [B + 1] first scratch page per widened request (E4M3 pools)
};

struct pa_plan {
  int B, Hq, Hkv, D, ps, C, G;
  int device, n_sm;
  float scale;
  int num_pages;
  int num_splits;   // 0 auto, 1 off, n forced
  int S_max;
  int max_items;
  int tpb, box_h, BN;
  // workspace
  void* ws;
  size_t ws_bytes;
  pa::WsHeader* hdr;           // set 0's header: holds the status word of every run
  SchedBufs sb[2];
  unsigned run_par;            // set used by the next pa_run
  int max_items2;
  bool use_pairs;             // head_dim <= 128: prefill runs on the two-stage kernel
  int last_launches;          // kernels the last pa_run enqueued
  int box_h2;                 // page box height of the two-stage kernel
  float* part_lse;
  float* part_o;
  // attention-kernel timing (pa_profile_*)
  cudaEvent_t* prof_ev;
  int prof_cap, prof_n, prof_on;
  // tensor-map cache
  const void* tm_ptr[4];       // q, k_pool, v_pool, out the maps were encoded for
  int tm_num_pages;
  CUtensorMap tm_q, tm_k, tm_v;
  CUtensorMap tm_o;            // out, box (32, G, 32 / G), 64-byte swizzle
  int use_dec;                 // decode kernel: -1 head_dim 128 only (default), 1 128 and 256, 0 never
  int causal;                  // 1 (default): causal mask; 0: every row sees all of its keys
  int fused_merge;             // 1: the last split warp merges; 0 (default): merge kernel
  int tstride;                 // page-table row stride in int32 entries (default C)
  int o_tma;                   // tm_o is used (G divides 32)
  CUtensorMap tm_k2, tm_v2;   // page boxes of box_h2 rows
  int kv_fp8;                  // 1: the pools hold E4M3 codes
  float k_scale, v_scale;      // their per-tensor descales
  int tm_fp8;                  // the pool maps were encoded for E4M3 pools
  // E4M3 pools: requests with two or more query blocks are widened once per run
  // into a bf16 scratch pool of widen_cap pages (pa_widen_kernel) and run on
  // the bf16 one-stage kernel; allocated on the first run that needs it
  int widen_req;               // -1 automatic capacity (default), 0 never widen, n pages
  int widen_cap;               // pages of the allocated scratch pool (0: none yet)
  void* widen_buf;             // K pool, V pool, page table [B, C]
  void* kw;
  void* vw;
  int* spt;
  CUtensorMap tm_kw, tm_vw;    // the scratch pools, bf16 page boxes of box_h rows
};

namespace {

int kv_tile(int D) {
  return D == 64 ? pa::TileCfg<64>::BN : (D == 128 ? pa::TileCfg<128>::BN : pa::TileCfg<256>::BN);
}

// CTAs of the persistent attention grid: one or two per SM depending on D.
int attn_grid(int D, int n_sm) {
  const int c = D == 64 ? pa::TileCfg<64>::CTAS
                        : (D == 128 ? pa::TileCfg<128>::CTAS : pa::TileCfg<256>::CTAS);
  return c * n_sm;
}

int auto_smax(int B, int Hkv, int n_sm) {
  const long units = (long)B * Hkv;
  long s = (8L * n_sm + units - 1) / units;
  if (s > pa::kMaxSplits) s = pa::kMaxSplits;
  if (s < 1) s = 1;
  return (int)s;
}

// (Re)allocate the workspace for the plan's current S_max.
int alloc_workspace(pa_plan* p) {
  const int G = p->G;
  const long blocks_per_req = (long)(((long)p->C * p->ps + p->tpb - 1) / p->tpb);
  long per_req = blocks_per_req > p->S_max ? blocks_per_req : p->S_max;
  const long max_items = (long)p->B * p->Hkv * per_req;
  if (max_items > (1L << 30)) {
    set_err("pa: work list would need %ld items (batch * heads_kv * capacity too large)",
            max_items);
    return PA_ERR_UNSUPPORTED;
  }
  (void)G;
  // second list: query-block pairs (two-stage prefill) or the blocks of widened
  // requests (E4M3 pools)
  // (E4M3 pools never use pairs, and their list is the longer one)
  const long max_items2 = p->kv_fp8 ? (long)p->B * p->Hkv * blocks_per_req
                          : (p->use_pairs ? (long)p->B * p->Hkv * ((blocks_per_req + 1) / 2) : 0);
  const size_t n_part_rows = p->S_max > 1 ? (size_t)p->B * p->Hkv * p->S_max * pa::kBM : 0;
  size_t off = 0;
  size_t o_hdr[2], o_req[2], o_aux[2], o_uoff[2], o_split[2], o_items[2], o_uoff2[2],
      o_items2[2], o_cnt[2], o_wpre[2];
  o_hdr[0] = off; off = align_up(off + sizeof(pa::WsHeader), 256);
  o_hdr[1] = off; off = align_up(off + sizeof(pa::WsHeader), 256);
  const size_t zero_bytes = off;   // both headers start zeroed
  for (int k = 0; k < 2; ++k) {
    o_req[k] = off; off = align_up(off + sizeof(int4) * (size_t)p->B, 256);
    o_aux[k] = off; off = align_up(off + sizeof(int4) * (size_t)p->B, 256);
    o_uoff[k] = off; off = align_up(off + sizeof(int) * (size_t)(p->B + 1), 256);
    o_split[k] = off; off = align_up(off + sizeof(int) * (size_t)p->B, 256);
    o_items[k] = off; off = align_up(off + sizeof(pa::PackedItem) * (size_t)max_items, 256);
    o_uoff2[k] = off; off = align_up(off + sizeof(int) * (size_t)(p->B + 1), 256);
    o_items2[k] = off; off = align_up(off + sizeof(pa::PackedItem) * (size_t)max_items2, 256);
    o_cnt[k] = off;
    off = align_up(off + (p->S_max > 1 ? sizeof(int) * (size_t)p->B * p->Hkv : 0), 256);
    o_wpre[k] = off; off = align_up(off + sizeof(int) * (size_t)(p->B + 1), 256);
  }
  const size_t o_plse = off; off = align_up(off + sizeof(float) * n_part_rows, 256);
  const size_t o_po = off; off = align_up(off + sizeof(float) * n_part_rows * p->D, 256);
  void* ws = nullptr;
  cudaError_t e = cudaMalloc(&ws, off);
  if (e != cudaSuccess) {
    set_err("pa: cudaMalloc of %zu workspace bytes failed: %s", off, cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  e = cudaMemset(ws, 0, zero_bytes);
  if (e != cudaSuccess) {
    cudaFree(ws);
    set_err("pa: cudaMemset failed: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  if (p->ws) cudaFree(p->ws);
  p->ws = ws;
  p->ws_bytes = off;
  char* c = static_cast<char*>(ws);
  for (int k = 0; k < 2; ++k) {
    SchedBufs& b = p->sb[k];
    b.hdr = reinterpret_cast<pa::WsHeader*>(c + o_hdr[k]);
    b.req_info = reinterpret_cast<int4*>(c + o_req[k]);
    b.req_aux = reinterpret_cast<int4*>(c + o_aux[k]);
    b.unit_off = reinterpret_cast<int*>(c + o_uoff[k]);
    b.split_list = reinterpret_cast<int*>(c + o_split[k]);
    b.items = reinterpret_cast<pa::PackedItem*>(c + o_items[k]);
    b.unit_off2 = reinterpret_cast<int*>(c + o_uoff2[k]);
    b.items2 = reinterpret_cast<pa::PackedItem*>(c + o_items2[k]);
    b.split_cnt = p->S_max > 1 ? reinterpret_cast<int*>(c + o_cnt[k]) : nullptr;
    b.wpre = reinterpret_cast<int*>(c + o_wpre[k]);
  }
  p->hdr = p->sb[0].hdr;
  p->run_par = 0;
  p->max_items2 = (int)max_items2;
  p->part_lse = reinterpret_cast<float*>(c + o_plse);
  p->part_o = reinterpret_cast<float*>(c + o_po);
  p->max_items = (int)max_items;
  return PA_OK;
}

// The E4M3 decode kernel splits its launch registers between warpgroups with
// setmaxnreg (see DecCfg): a build whose kernel uses another launch count
// would leave the softmax warpgroup's increase unsatisfiable, so it is
// refused before any launch.
template <int D, int RR>
bool decode_f8_regs_ok(int* got) {
  cudaFuncAttributes a;
  if (cudaFuncGetAttributes(&a, pa::pa_decode_kernel<D, RR, true>) != cudaSuccess) return false;
  *got = a.numRegs;
  return a.numRegs == pa::DecCfg<D, pa::DecRows<RR>::NR, true>::LAUNCH_REGS;
}

template <int D>
int check_decode_f8_regs(const char* who) {
  int got = -1;
  const bool ok = decode_f8_regs_ok<D, 4>(&got) && decode_f8_regs_ok<D, 8>(&got) &&
                  decode_f8_regs_ok<D, 16>(&got) && decode_f8_regs_ok<D, 32>(&got);
  if (!ok) {
    set_err("%s: the E4M3 decode kernel for head_dim %d was built with %d registers per "
            "thread; its warpgroup register split needs exactly %d", who, D, got,
            pa::DecCfg<D, 16, true>::LAUNCH_REGS);
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

template <int D, int RR>
cudaError_t set_decode_smem_attr() {
  cudaError_t e = cudaFuncSetAttribute(pa::pa_decode_kernel<D, RR, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       pa::DecCfg<D, pa::DecRows<RR>::NR, false>::SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(pa::pa_decode_kernel<D, RR, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pa::DecCfg<D, pa::DecRows<RR>::NR, true>::SMEM_BYTES);
  return e;
}

template <int D>
cudaError_t set_smem_attr() {
  cudaError_t e = cudaFuncSetAttribute(pa::pa_attention_kernel<D, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       pa::TileCfg<D, false>::SMEM_BYTES);
  if constexpr (D >= 128) {
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(pa::pa_attention_kernel<D, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               pa::TileCfg<D, true>::SMEM_BYTES);
  }
  if constexpr (D <= 128) {
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(pa::pa_pair_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               pa::PairCfg<D>::SMEM_BYTES);
  }
  if constexpr (D >= 128) {
    if (e == cudaSuccess) e = set_decode_smem_attr<D, 4>();
    if (e == cudaSuccess) e = set_decode_smem_attr<D, 8>();
    if (e == cudaSuccess) e = set_decode_smem_attr<D, 16>();
    if (e == cudaSuccess) e = set_decode_smem_attr<D, 32>();
  }
  return e;
}

// Decode-only runs: G query rows per (request, KV head), RR = G rounded up;
// F8: E4M3 pools.
template <int D, int RR, bool F8>
cudaError_t launch_decode_rr(int n_sm, cudaStream_t st, const CUtensorMap& tk,
                             const CUtensorMap& tv, const pa::AttnParams& ap) {
  using C = pa::DecCfg<D, pa::DecRows<RR>::NR, F8>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_sm);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa::pa_decode_kernel<D, RR, F8>, tk, tv, ap);
}

template <int D, bool F8>
cudaError_t launch_decode_d(int G, int n_sm, cudaStream_t st, const CUtensorMap& tk,
                            const CUtensorMap& tv, const pa::AttnParams& ap) {
  if (G <= 4) return launch_decode_rr<D, 4, F8>(n_sm, st, tk, tv, ap);
  if (G <= 8) return launch_decode_rr<D, 8, F8>(n_sm, st, tk, tv, ap);
  if (G <= 16) return launch_decode_rr<D, 16, F8>(n_sm, st, tk, tv, ap);
  return launch_decode_rr<D, 32, F8>(n_sm, st, tk, tv, ap);
}

cudaError_t launch_decode(int D, int G, bool fp8, int n_sm, cudaStream_t st,
                          const CUtensorMap& tk, const CUtensorMap& tv, const pa::AttnParams& ap) {
  if (fp8)
    return D == 128 ? launch_decode_d<128, true>(G, n_sm, st, tk, tv, ap)
                    : launch_decode_d<256, true>(G, n_sm, st, tk, tv, ap);
  return D == 128 ? launch_decode_d<128, false>(G, n_sm, st, tk, tv, ap)
                  : launch_decode_d<256, false>(G, n_sm, st, tk, tv, ap);
}

template <int D>
cudaError_t launch_pairs(int n_sm, cudaStream_t st, const CUtensorMap& tq, const CUtensorMap& tk,
                         const CUtensorMap& tv, const CUtensorMap& to, const pa::AttnParams& ap) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_sm);
  cfg.blockDim = dim3(pa::PairCfg<D>::THREADS);
  cfg.dynamicSmemBytes = pa::PairCfg<D>::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa::pa_pair_kernel<D>, tq, tk, tv, to, ap);
}

// The attention kernel and the merge are programmatic dependents of the
// kernel launched before them on the stream (their prologues overlap it; each
// waits with griddepcontrol.wait before reading its results).
template <int D, bool F8>
cudaError_t launch_attention(int n_sm, cudaStream_t st, const CUtensorMap& tq,
                             const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, const pa::AttnParams& ap) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pa::TileCfg<D, F8>::CTAS * n_sm);
  cfg.blockDim = dim3(pa::TileCfg<D, F8>::THREADS);
  cfg.dynamicSmemBytes = pa::TileCfg<D, F8>::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa::pa_attention_kernel<D, F8>, tq, tk, tv, to, ap);
}

// fp8: E4M3 pools (head_dim 128 or 256; pa_set_kv_fp8 refuses 64)
cudaError_t launch_attention_d(int D, bool fp8, int n_sm, cudaStream_t st, const CUtensorMap& tq,
                               const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& to, const pa::AttnParams& ap) {
  if (fp8)
    return D == 128 ? launch_attention<128, true>(n_sm, st, tq, tk, tv, to, ap)
                    : launch_attention<256, true>(n_sm, st, tq, tk, tv, to, ap);
  switch (D) {
    case 64: return launch_attention<64, false>(n_sm, st, tq, tk, tv, to, ap);
    case 128: return launch_attention<128, false>(n_sm, st, tq, tk, tv, to, ap);
    default: return launch_attention<256, false>(n_sm, st, tq, tk, tv, to, ap);
  }
}

// The scheduler is a programmatic dependent of the kernel before it (the
// previous run's attention or merge kernel): it builds this run's work list in
// the other set of buffers while that kernel finishes, and waits for it
// (griddepcontrol.wait) before it exits, so everything launched after the
// scheduler is ordered after the previous run.
cudaError_t launch_schedule(cudaStream_t st, const pa::SchedParams& sp) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(pa::kCostBuckets);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa::pa_schedule_kernel, sp);
}

cudaError_t launch_merge(int n_sm, cudaStream_t st, const pa::MergeParams& mp) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * n_sm);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa::pa_merge_kernel, mp);
}

int encode(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims,
           const cuuint64_t* strides, const cuuint32_t* box, const char* what,
           CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B,
           CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    set_err("pa: cuTensorMapEncodeTiled is not available from the driver");
    return PA_ERR_CUDA;
  }
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, dt, rank, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_err("pa: cuTensorMapEncodeTiled(%s) failed with %d", what, (int)r);
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

int build_maps(pa_plan* p, const void* q, const void* k, const void* v, void* out) {
  if (p->tm_ptr[0] == q && p->tm_ptr[1] == k && p->tm_ptr[2] == v && p->tm_ptr[3] == out &&
      p->tm_num_pages == p->num_pages && p->tm_fp8 == p->kv_fp8)
    return PA_OK;
  const cuuint64_t e = 2;  // bytes per bf16
  // q [T, Hq, D]: dims (D, Hq, T bound); box (64, G, tokens per block).
  // T is only known on the device; every coordinate the kernel issues stays
  // below cu_q_lens[B], and B * C * ps bounds T for valid inputs.
  {
    cuuint64_t tb = (cuuint64_t)p->B * p->C * p->ps;
    cuuint64_t dims[3] = {(cuuint64_t)p->D, (cuuint64_t)p->Hq, tb};
    cuuint64_t str[2] = {(cuuint64_t)p->D * e, (cuuint64_t)p->Hq * p->D * e};
    cuuint32_t box[3] = {64, (cuuint32_t)p->G, (cuuint32_t)p->tpb};
    int rc = encode(&p->tm_q, q, 3, dims, str, box, "q");
    if (rc) return rc;
    // out has q's layout; a softmax warp stores its 32 rows = 32 / G whole tokens
    p->o_tma = (32 % p->G == 0) ? 1 : 0;
    if (p->o_tma) {
      cuuint32_t obox[3] = {32, (cuuint32_t)p->G, (cuuint32_t)(32 / p->G)};
      rc = encode(&p->tm_o, out, 3, dims, str, obox, "out", CU_TENSOR_MAP_SWIZZLE_64B);
      if (rc) return rc;
    }
  }
  // E4M3 pools [P, ps, Hkv, D] bytes: dims (D, Hkv, ps, P); box (128, 1, box_h, 1),
  // 128-byte swizzle (D / 128 boxes per page part)
  if (p->kv_fp8) {
    cuuint64_t P = p->num_pages > 0 ? (cuuint64_t)p->num_pages : (cuuint64_t)0x7fffffff;
    cuuint64_t dims[4] = {(cuuint64_t)p->D, (cuuint64_t)p->Hkv, (cuuint64_t)p->ps, P};
    cuuint64_t str[3] = {(cuuint64_t)p->D, (cuuint64_t)p->Hkv * p->D,
                         (cuuint64_t)p->ps * p->Hkv * p->D};
    cuuint32_t box[4] = {128, 1, (cuuint32_t)p->box_h, 1};
    int rc = encode(&p->tm_k, k, 4, dims, str, box, "k_pool (e4m3)", CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_DATA_TYPE_UINT8);
    if (rc) return rc;
    rc = encode(&p->tm_v, v, 4, dims, str, box, "v_pool (e4m3)", CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_DATA_TYPE_UINT8);
    if (rc) return rc;
  } else {
    // pools [P, ps, Hkv, D]: dims (D, Hkv, ps, P); box (64, 1, box_h, 1).
    cuuint64_t P = p->num_pages > 0 ? (cuuint64_t)p->num_pages : (cuuint64_t)0x7fffffff;
    cuuint64_t dims[4] = {(cuuint64_t)p->D, (cuuint64_t)p->Hkv, (cuuint64_t)p->ps, P};
    cuuint64_t str[3] = {(cuuint64_t)p->D * e, (cuuint64_t)p->Hkv * p->D * e,
                         (cuuint64_t)p->ps * p->Hkv * p->D * e};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)p->box_h, 1};
    int rc = encode(&p->tm_k, k, 4, dims, str, box, "k_pool");
    if (rc) return rc;
    rc = encode(&p->tm_v, v, 4, dims, str, box, "v_pool");
    if (rc) return rc;
    if (p->use_pairs) {
      cuuint32_t box2[4] = {64, 1, (cuuint32_t)p->box_h2, 1};
      rc = encode(&p->tm_k2, k, 4, dims, str, box2, "k_pool");
      if (rc) return rc;
      rc = encode(&p->tm_v2, v, 4, dims, str, box2, "v_pool");
      if (rc) return rc;
    }
  }
  p->tm_ptr[0] = q;
  p->tm_ptr[1] = k;
  p->tm_ptr[2] = v;
  p->tm_ptr[3] = out;
  p->tm_num_pages = p->num_pages;
  p->tm_fp8 = p->kv_fp8;
  return PA_OK;
}

bool aligned16(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }

// Automatic scratch capacity for widened E4M3 requests: every page the batch
// can hold, up to 512 MiB of bf16 K and V.
constexpr size_t kWidenAutoBytes = size_t(512) << 20;

void free_widen(pa_plan* p) {
  if (p->widen_buf) cudaFree(p->widen_buf);
  p->widen_buf = p->kw = p->vw = nullptr;
  p->spt = nullptr;
  p->widen_cap = 0;
}

// Allocate the scratch pools and page table of widened requests and encode
// their tensor maps ([cap, ps, Hkv, D] bf16, the bf16 pools' page boxes).
int alloc_widen(pa_plan* p) {
  const size_t part = (size_t)p->ps * p->Hkv * p->D * 2;   // bytes of one bf16 page part
  const long all = (long)p->B * p->C;
  long cap = p->widen_req > 0 ? p->widen_req : (long)(kWidenAutoBytes / (2 * part));
  if (cap > all) cap = all;
  if (cap < 1) cap = 1;
  const size_t o_v = align_up(part * (size_t)cap, 256);
  const size_t o_t = o_v + align_up(part * (size_t)cap, 256);
  const size_t bytes = o_t + sizeof(int) * (size_t)all;
  void* buf = nullptr;
  cudaError_t e = cudaMalloc(&buf, bytes);
  if (e != cudaSuccess) {
    set_err("cudaMalloc of %zu bytes for the widened E4M3 pages failed: %s "
            "(pa_set_kv_fp8_widen sets a smaller capacity, or 0 for none)",
            bytes, cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  free_widen(p);
  p->widen_buf = buf;
  p->kw = buf;
  p->vw = static_cast<char*>(buf) + o_v;
  p->spt = reinterpret_cast<int*>(static_cast<char*>(buf) + o_t);
  const cuuint64_t e2 = 2;
  cuuint64_t dims[4] = {(cuuint64_t)p->D, (cuuint64_t)p->Hkv, (cuuint64_t)p->ps, (cuuint64_t)cap};
  cuuint64_t str[3] = {(cuuint64_t)p->D * e2, (cuuint64_t)p->Hkv * p->D * e2,
                       (cuuint64_t)p->ps * p->Hkv * p->D * e2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)p->box_h, 1};
  int rc = encode(&p->tm_kw, p->kw, 4, dims, str, box, "widened k");
  if (rc == PA_OK) rc = encode(&p->tm_vw, p->vw, 4, dims, str, box, "widened v");
  if (rc != PA_OK) {
    free_widen(p);
    return rc;
  }
  p->widen_cap = (int)cap;
  return PA_OK;
}

cudaError_t launch_widen(int n_sm, cudaStream_t st, const pa::WidenParams& wp) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(4 * n_sm);
  cfg.blockDim = dim3(pa::kWidenThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa::pa_widen_kernel, wp);
}

}  // namespace

extern "C" {

const char* pa_last_error(void) { return g_err; }

pa_plan* pa_create_plan(int batch, int heads_q, int heads_kv, int head_dim, int page_size,
                        int capacity) {
  g_err[0] = 0;
  if (batch <= 0 || heads_q <= 0 || heads_kv <= 0 || head_dim <= 0 || page_size <= 0 ||
      capacity <= 0) {
    set_err("pa_create_plan: every argument must be > 0 (batch=%d heads_q=%d heads_kv=%d "
            "head_dim=%d page_size=%d capacity=%d)",
            batch, heads_q, heads_kv, head_dim, page_size, capacity);
    return nullptr;
  }
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) {
    set_err("pa_create_plan: unsupported head_dim %d (supported: 64, 128, 256)", head_dim);
    return nullptr;
  }
  if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128) {
    set_err("pa_create_plan: unsupported page_size %d (supported: 16, 32, 64, 128)", page_size);
    return nullptr;
  }
  if (heads_q % heads_kv != 0) {
    set_err("pa_create_plan: heads_q %d is not a multiple of heads_kv %d", heads_q, heads_kv);
    return nullptr;
  }
  const int G = heads_q / heads_kv;
  if (G > 32) {
    set_err("pa_create_plan: GQA ratio %d exceeds 32", G);
    return nullptr;
  }
  if ((long)capacity * page_size > (1L << 30)) {
    set_err("pa_create_plan: capacity * page_size too large");
    return nullptr;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  int n_sm = 0, major = 0;
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) {
    set_err("pa_create_plan: no usable CUDA device: %s", cudaGetErrorString(e));
    return nullptr;
  }
  if (major != 10) {
    set_err("pa_create_plan: device %d has compute capability %d.x; this library is built "
            "for sm_100a only", dev, major);
    return nullptr;
  }
  if (head_dim == 64) e = set_smem_attr<64>();
  else if (head_dim == 128) e = set_smem_attr<128>();
  else e = set_smem_attr<256>();
  if (e != cudaSuccess) {
    set_err("pa_create_plan: cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
    return nullptr;
  }
  if ((head_dim == 128 && check_decode_f8_regs<128>("pa_create_plan") != PA_OK) ||
      (head_dim == 256 && check_decode_f8_regs<256>("pa_create_plan") != PA_OK))
    return nullptr;
  pa_plan* p = new pa_plan();
  p->B = batch; p->Hq = heads_q; p->Hkv = heads_kv; p->D = head_dim; p->ps = page_size;
  p->C = capacity; p->G = G; p->device = dev; p->n_sm = n_sm;
  p->scale = 1.0f / std::sqrt((float)head_dim);
  p->num_pages = 0;
  p->num_splits = 0;
  p->BN = kv_tile(head_dim);
  p->tpb = pa::kBM / G;
  p->box_h = page_size < p->BN ? page_size : p->BN;
  p->use_pairs = false;       // pa_set_two_stage_prefill turns it on (head_dim <= 128)
  p->last_launches = 2;
  p->box_h2 = page_size < pa::PairCfg<128>::BN ? page_size : pa::PairCfg<128>::BN;
  p->S_max = auto_smax(batch, heads_kv, n_sm);
  p->ws = nullptr;
  p->prof_ev = nullptr;
  p->prof_cap = p->prof_n = p->prof_on = 0;
  p->tm_ptr[0] = p->tm_ptr[1] = p->tm_ptr[2] = p->tm_ptr[3] = nullptr;
  p->o_tma = 0;
  p->use_dec = -1;
  p->causal = 1;
  p->fused_merge = 0;
  p->tstride = p->C;
  p->kv_fp8 = 0;
  p->k_scale = p->v_scale = 1.0f;
  p->tm_fp8 = 0;
  p->tm_num_pages = -1;
  p->widen_req = -1;
  p->widen_cap = 0;
  p->widen_buf = p->kw = p->vw = nullptr;
  p->spt = nullptr;
  if (alloc_workspace(p) != PA_OK) {
    delete p;
    return nullptr;
  }
  return p;
}

static void free_profile_events(pa_plan* p) {
  if (p->prof_ev) {
    for (int i = 0; i < 2 * p->prof_cap; ++i) cudaEventDestroy(p->prof_ev[i]);
    delete[] p->prof_ev;
  }
  p->prof_ev = nullptr;
  p->prof_cap = p->prof_n = p->prof_on = 0;
}

void pa_destroy(pa_plan* p) {
  if (!p) return;
  free_profile_events(p);
  free_widen(p);
  if (p->ws) cudaFree(p->ws);
  delete p;
}

int pa_set_scale(pa_plan* p, float scale) {
  if (!p) { set_err("pa_set_scale: NULL plan"); return PA_ERR_INVALID; }
  if (!(scale > 0.f) || !std::isfinite(scale)) {
    set_err("pa_set_scale: scale must be finite and > 0");
    return PA_ERR_INVALID;
  }
  p->scale = scale;
  return PA_OK;
}

int pa_set_num_pages(pa_plan* p, int num_pages) {
  if (!p) { set_err("pa_set_num_pages: NULL plan"); return PA_ERR_INVALID; }
  if (num_pages < 0) { set_err("pa_set_num_pages: negative page count"); return PA_ERR_INVALID; }
  p->num_pages = num_pages;
  return PA_OK;
}

int pa_set_num_splits(pa_plan* p, int num_splits) {
  if (!p) { set_err("pa_set_num_splits: NULL plan"); return PA_ERR_INVALID; }
  if (num_splits < 0 || num_splits > pa::kMaxSplits) {
    set_err("pa_set_num_splits: %d outside [0, %d]", num_splits, pa::kMaxSplits);
    return PA_ERR_INVALID;
  }
  int want = num_splits == 0 ? auto_smax(p->B, p->Hkv, p->n_sm) : num_splits;
  if (want != p->S_max) {
    const int old = p->S_max;
    p->S_max = want;
    int rc = alloc_workspace(p);
    if (rc != PA_OK) {
      p->S_max = old;
      return rc;
    }
  }
  p->num_splits = num_splits;
  return PA_OK;
}

size_t pa_workspace_bytes(const pa_plan* p) { return p ? p->ws_bytes : 0; }

int pa_max_splits(const pa_plan* p) { return p ? p->S_max : 0; }

int pa_get_status(pa_plan* p, pa_stream_t stream, uint32_t* status, int clear) {
  if (!p || !status) { set_err("pa_get_status: NULL argument"); return PA_ERR_INVALID; }
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess) e = cudaMemcpy(status, &p->hdr->status, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && clear) e = cudaMemset(&p->hdr->status, 0, sizeof(uint32_t));
  if (e != cudaSuccess) {
    set_err("pa_get_status: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

int pa_run(pa_plan* p, const void* q, const void* k_pool, const void* v_pool,
           const int32_t* page_table, const int32_t* seq_lens, const int32_t* cu_q_lens,
           void* out, float* lse, pa_stream_t stream) {
  if (!p) { set_err("pa_run: NULL plan"); return PA_ERR_INVALID; }
  if (!q || !k_pool || !v_pool || !page_table || !seq_lens || !out) {
    set_err("pa_run: NULL pointer (q, k_pool, v_pool, page_table, seq_lens and out are required)");
    return PA_ERR_INVALID;
  }
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out) ||
      !aligned16(page_table) || !aligned16(seq_lens) || (cu_q_lens && !aligned16(cu_q_lens)) ||
      (lse && !aligned16(lse))) {
    set_err("pa_run: every pointer must be 16-byte aligned");
    return PA_ERR_INVALID;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device) {
    set_err("pa_run: current device %d is not the plan's device %d", dev, p->device);
    return PA_ERR_INVALID;
  }
  int rc = build_maps(p, q, k_pool, v_pool, out);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  // this run's set of scheduler outputs (the previous run may still read the other)
  const SchedBufs& bufs = p->sb[p->run_par & 1u];
  pa::SchedParams sp = {};
  sp.seq_lens = seq_lens;
  sp.cu_q_lens = cu_q_lens;
  sp.items = bufs.items;
  sp.req_info = bufs.req_info;
  sp.req_aux = bufs.req_aux;
  sp.unit_off = bufs.unit_off;
  sp.split_list = bufs.split_list;
  // without cu_q_lens every request is one decode token: no query-block pairs;
  // the two-stage kernel reads bf16 pools only, so E4M3 pools skip it too
  const bool pairs = p->use_pairs && cu_q_lens != nullptr && !p->kv_fp8;
  // E4M3 pools with query blocks: requests of two or more blocks are widened
  // once (pa_widen_kernel) and run on the bf16 kernel from the second list
  // (the scratch pool is allocated by pa_set_kv_fp8 / pa_set_kv_fp8_widen;
  // pa_run allocates nothing)
  const bool wide = p->kv_fp8 && cu_q_lens != nullptr && p->widen_buf != nullptr;
  sp.items2 = (pairs || wide) ? bufs.items2 : nullptr;
  sp.wide_cap = wide ? p->widen_cap : 0;
  sp.wpre = bufs.wpre;
  sp.unit_off2 = bufs.unit_off2;
  sp.max_items2 = p->max_items2;
  sp.hdr = bufs.hdr;
  sp.status = &p->hdr->status;
  sp.max_items = p->max_items;
  sp.B = p->B; sp.Hkv = p->Hkv; sp.G = p->G; sp.C = p->C; sp.ps = p->ps; sp.BN = p->BN;
  sp.tpb = p->tpb;
  sp.causal = p->causal;
  sp.S_max = p->num_splits == 1 ? 1 : p->S_max;
  const bool fused = p->fused_merge && sp.S_max > 1;
  sp.split_cnt = fused ? bufs.split_cnt : nullptr;
  sp.forced_splits = p->num_splits > 1 ? p->num_splits : 0;
  // decode-only runs (one query token per request) with up to 32 query heads
  // per KV head go to the keys-as-M decode kernel (one CTA per SM): by default
  // at head_dim 128, on request at 256 too; the same rule for E4M3 pools
  const bool dec_shape = p->G <= 32 &&
                         ((p->use_dec == -1 && p->D == 128) || (p->use_dec == 1 && p->D >= 128));
  const bool dec = cu_q_lens == nullptr && dec_shape;
  // E4M3 pools with cu_q_lens: rows of one query token (the decode rows of a
  // mixed batch) run on the E4M3 decode kernel from a second segment of the
  // main list; on the one-stage kernel each would widen its tiles through one
  // warp (bf16 pools keep one launch: there the one-stage kernel overlaps the
  // decode rows' HBM streaming with the prefill blocks' tensor work)
  const bool dec_seg = p->kv_fp8 && cu_q_lens != nullptr && dec_shape;
  sp.split_decode = dec_seg ? 1 : 0;
  sp.n_ctas = dec ? p->n_sm : attn_grid(p->D, p->n_sm);
  cudaError_t le = launch_schedule(st, sp);

  pa::AttnParams ap = {};
  ap.q = static_cast<const uint16_t*>(q);
  ap.page_table = page_table;
  ap.cu_q_lens = cu_q_lens;
  ap.out = static_cast<uint16_t*>(out);
  ap.lse = lse;
  ap.items = bufs.items;
  ap.hdr = bufs.hdr;
  ap.part_o = p->part_o;
  ap.part_lse = p->part_lse;
  ap.status = &p->hdr->status;
  ap.B = p->B; ap.Hq = p->Hq; ap.Hkv = p->Hkv; ap.G = p->G; ap.C = p->C; ap.ps = p->ps;
  ap.num_pages = p->num_pages;
  ap.S_max = p->S_max;
  ap.tpb = p->tpb;
  ap.box_h = p->box_h;
  ap.ps_log2 = __builtin_ctz((unsigned)p->ps);
  ap.box_log2 = __builtin_ctz((unsigned)p->box_h);
  ap.tstride = p->tstride;
  ap.causal = p->causal;
  ap.o_tma = p->o_tma;
  ap.split_cnt = bufs.split_cnt;
  ap.fused_merge = fused ? 1 : 0;
  ap.scale_log2 = p->scale * 1.4426950408889634f * (p->kv_fp8 ? p->k_scale : 1.0f);
  ap.v_scale = p->kv_fp8 ? p->v_scale : 1.0f;
  const bool prof = p->prof_on && p->prof_n < p->prof_cap;
  if (prof) cudaEventRecord(p->prof_ev[2 * p->prof_n], st);
  if (le == cudaSuccess && pairs) {
    // query-block pairs (prefill) first, on the two-stage kernel
    pa::AttnParams ap2 = ap;
    ap2.items = bufs.items2;
    ap2.box_h = p->box_h2;
    ap2.box_log2 = __builtin_ctz((unsigned)p->box_h2);
    le = p->D == 64 ? launch_pairs<64>(p->n_sm, st, p->tm_q, p->tm_k2, p->tm_v2, p->tm_o, ap2)
                    : launch_pairs<128>(p->n_sm, st, p->tm_q, p->tm_k2, p->tm_v2, p->tm_o, ap2);
  }
  if (le == cudaSuccess && wide) {
    // widen the chosen requests' pages, then run their blocks over the
    // scratch pools as a bf16 batch (descales still in scale_log2 and v_scale)
    pa::WidenParams wp;
    wp.k8 = static_cast<const uint4*>(k_pool);
    wp.v8 = static_cast<const uint4*>(v_pool);
    wp.k16 = static_cast<uint4*>(p->kw);
    wp.v16 = static_cast<uint4*>(p->vw);
    wp.spt = p->spt;
    wp.page_table = page_table;
    wp.wpre = bufs.wpre;
    wp.hdr = bufs.hdr;
    wp.status = &p->hdr->status;
    wp.B = p->B; wp.C = p->C; wp.tstride = p->tstride; wp.num_pages = p->num_pages;
    wp.part_u4 = p->ps * p->Hkv * p->D / 16;
    le = launch_widen(p->n_sm, st, wp);
    if (le == cudaSuccess) {
      pa::AttnParams aw = ap;
      aw.items = bufs.items2;
      aw.list = 1;
      aw.page_table = p->spt;
      aw.tstride = p->C;
      aw.num_pages = p->widen_cap;
      le = launch_attention_d(p->D, false, p->n_sm, st, p->tm_q, p->tm_kw, p->tm_vw, p->tm_o, aw);
    }
  }
  if (le == cudaSuccess)
    le = dec ? launch_decode(p->D, p->G, p->kv_fp8 != 0, p->n_sm, st, p->tm_k, p->tm_v, ap)
             : launch_attention_d(p->D, p->kv_fp8 != 0, p->n_sm, st, p->tm_q, p->tm_k, p->tm_v,
                                  p->tm_o, ap);
  if (le == cudaSuccess && dec_seg) {
    pa::AttnParams ad = ap;
    ad.list = 2;
    le = launch_decode(p->D, p->G, true, p->n_sm, st, p->tm_k, p->tm_v, ad);
  }
  if (prof) {
    cudaEventRecord(p->prof_ev[2 * p->prof_n + 1], st);
    ++p->prof_n;
  }
  if (le == cudaSuccess && sp.S_max > 1 && !fused) {
    pa::MergeParams mp;
    mp.req_info = bufs.req_info;
    mp.split_list = bufs.split_list;
    mp.hdr = bufs.hdr;
    mp.part_o = p->part_o;
    mp.part_lse = p->part_lse;
    mp.out = static_cast<uint16_t*>(out);
    mp.lse = lse;
    mp.B = p->B; mp.Hq = p->Hq; mp.Hkv = p->Hkv; mp.G = p->G; mp.D = p->D; mp.S_max = p->S_max;
    le = launch_merge(p->n_sm, st, mp);
  }
  if (le != cudaSuccess) {
    set_err("pa_run: launch failed: %s", cudaGetErrorString(le));
    return PA_ERR_CUDA;
  }
  p->last_launches = 2 + (pairs ? 1 : 0) + (wide ? 2 : 0) + (dec_seg ? 1 : 0) +
                     (sp.S_max > 1 && !fused ? 1 : 0);
  p->run_par ^= 1u;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_err("pa_run: launch failed: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

int pa_append_kv(pa_plan* p, const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                 const int32_t* page_table, const int32_t* seq_lens, const int32_t* cu_q_lens,
                 pa_stream_t stream) {
  if (!p) { set_err("pa_append_kv: NULL plan"); return PA_ERR_INVALID; }
  if (!k_new || !v_new || !k_pool || !v_pool || !page_table || !seq_lens) {
    set_err("pa_append_kv: NULL pointer (k_new, v_new, k_pool, v_pool, page_table and "
            "seq_lens are required)");
    return PA_ERR_INVALID;
  }
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool) ||
      !aligned16(page_table) || !aligned16(seq_lens) || (cu_q_lens && !aligned16(cu_q_lens))) {
    set_err("pa_append_kv: every pointer must be 16-byte aligned");
    return PA_ERR_INVALID;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device) {
    set_err("pa_append_kv: current device %d is not the plan's device %d", dev, p->device);
    return PA_ERR_INVALID;
  }
  pa::AppendParams ap;
  ap.k_new = static_cast<const uint4*>(k_new);
  ap.v_new = static_cast<const uint4*>(v_new);
  ap.k_pool = static_cast<uint4*>(k_pool);
  ap.v_pool = static_cast<uint4*>(v_pool);
  ap.page_table = page_table;
  ap.seq_lens = seq_lens;
  ap.cu_q_lens = cu_q_lens;
  ap.status = &p->hdr->status;
  ap.B = p->B; ap.C = p->C; ap.ps = p->ps; ap.num_pages = p->num_pages;
  ap.tstride = p->tstride;
  ap.row_u4 = p->Hkv * p->D / 8;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // one warp per new token; T is known only on the device, so the grid is
  // sized for the most tokens the batch can hold (B * C * ps), at most four
  // CTAs of eight warps per SM
  const long max_tok = (long)p->B * p->C * p->ps;
  const long want = (max_tok + (pa::kAppendThreads / 32) - 1) / (pa::kAppendThreads / 32);
  const int grid = (int)(want < 4L * p->n_sm ? want : 4L * p->n_sm);
  pa::pa_append_kernel<<<grid, pa::kAppendThreads, 0, st>>>(ap);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_err("pa_append_kv: launch failed: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

int pa_set_fused_merge(pa_plan* p, int on) {
  if (!p) { set_err("pa_set_fused_merge: NULL plan"); return PA_ERR_INVALID; }
  p->fused_merge = on ? 1 : 0;
  return PA_OK;
}

int pa_set_causal(pa_plan* p, int causal) {
  if (!p) { set_err("pa_set_causal: NULL plan"); return PA_ERR_INVALID; }
  p->causal = causal ? 1 : 0;
  return PA_OK;
}

int pa_set_page_table_stride(pa_plan* p, int row_stride) {
  if (!p) { set_err("pa_set_page_table_stride: NULL plan"); return PA_ERR_INVALID; }
  if (row_stride < p->C) {
    set_err("pa_set_page_table_stride: row stride %d must be >= capacity %d", row_stride, p->C);
    return PA_ERR_INVALID;
  }
  p->tstride = row_stride;
  return PA_OK;
}

int pa_selftest_wait_timeout(uint32_t limit_us, uint32_t* status_out,
                             uint32_t* elapsed_us_out) {
  if (!status_out || !elapsed_us_out) {
    set_err("pa_selftest_wait_timeout: NULL argument");
    return PA_ERR_INVALID;
  }
  if (limit_us < 1 || limit_us > 1000000) {
    set_err("pa_selftest_wait_timeout: limit_us %u outside [1, 1000000]", limit_us);
    return PA_ERR_INVALID;
  }
  unsigned* d = nullptr;   // [0] status, [1..2] elapsed microseconds of warps 1 and 2
  cudaError_t e = cudaMalloc(&d, 3 * sizeof(unsigned));
  if (e == cudaSuccess) e = cudaMemset(d, 0, 3 * sizeof(unsigned));
  if (e == cudaSuccess) {
    pa::pa_selftest_wait_kernel<<<1, 96>>>(d, (uint64_t)limit_us * 1000u, d + 1);
    e = cudaGetLastError();
  }
  unsigned h[3] = {0, 0, 0};
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(h, d, sizeof h, cudaMemcpyDeviceToHost);
  if (d) cudaFree(d);
  if (e != cudaSuccess) {
    set_err("pa_selftest_wait_timeout: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  *status_out = h[0];
  elapsed_us_out[0] = h[1];
  elapsed_us_out[1] = h[2];
  return PA_OK;
}

int pa_set_kv_fp8(pa_plan* p, int on, float k_scale, float v_scale) {
  if (!p) { set_err("pa_set_kv_fp8: NULL plan"); return PA_ERR_INVALID; }
  if (!on) {
    if (p->kv_fp8) {
      p->kv_fp8 = 0;
      int rc = alloc_workspace(p);   // the second list shrinks back
      if (rc != PA_OK) { p->kv_fp8 = 1; return rc; }
      free_widen(p);
    }
    p->k_scale = p->v_scale = 1.0f;
    return PA_OK;
  }
  if (!(k_scale > 0.f) || !std::isfinite(k_scale) || !(v_scale > 0.f) || !std::isfinite(v_scale)) {
    set_err("pa_set_kv_fp8: descales must be finite and > 0 (k_scale=%g v_scale=%g)",
            (double)k_scale, (double)v_scale);
    return PA_ERR_INVALID;
  }
  if (p->D != 128 && p->D != 256) {
    set_err("pa_set_kv_fp8: head_dim %d has no E4M3 kernels (128 and 256 only)", p->D);
    return PA_ERR_UNSUPPORTED;
  }
  if (!p->kv_fp8) {
    p->kv_fp8 = 1;
    int rc = alloc_workspace(p);     // room for the blocks of widened requests
    if (rc == PA_OK && p->widen_req != 0) {
      rc = alloc_widen(p);           // the scratch pool of widened requests
      if (rc != PA_OK) {
        p->kv_fp8 = 0;
        alloc_workspace(p);          // back to the bf16 sizes (smaller: cannot fail on memory)
        return rc;
      }
    }
    if (rc != PA_OK) { p->kv_fp8 = 0; return rc; }
  }
  p->k_scale = k_scale;
  p->v_scale = v_scale;
  return PA_OK;
}

int pa_set_kv_fp8_widen(pa_plan* p, int max_pages) {
  if (!p) { set_err("pa_set_kv_fp8_widen: NULL plan"); return PA_ERR_INVALID; }
  if (max_pages < -1) {
    set_err("pa_set_kv_fp8_widen: max_pages %d (use -1, 0 or a page count)", max_pages);
    return PA_ERR_INVALID;
  }
  if (max_pages != p->widen_req) {
    free_widen(p);
    p->widen_req = max_pages;
    if (p->kv_fp8 && max_pages != 0) {
      int rc = alloc_widen(p);       // the new capacity, now
      if (rc != PA_OK) return rc;    // (the plan then widens nothing)
    }
  }
  return PA_OK;
}

int pa_set_decode_kernel(pa_plan* p, int on) {
  if (!p) { set_err("pa_set_decode_kernel: NULL plan"); return PA_ERR_INVALID; }
  p->use_dec = on ? 1 : 0;
  return PA_OK;
}

int pa_set_two_stage_prefill(pa_plan* p, int on) {
  if (!p) { set_err("pa_set_two_stage_prefill: NULL plan"); return PA_ERR_INVALID; }
  if (on && p->D > 128) {
    set_err("pa_set_two_stage_prefill: head_dim %d has no two-stage kernel (64 and 128 only)",
            p->D);
    return PA_ERR_UNSUPPORTED;
  }
  const bool want = on != 0;
  if (want != p->use_pairs) {
    const bool old = p->use_pairs;
    p->use_pairs = want;
    int rc = alloc_workspace(p);
    if (rc != PA_OK) {
      p->use_pairs = old;
      return rc;
    }
    p->tm_num_pages = -1;   // rebuild tensor maps (two-stage boxes)
  }
  return PA_OK;
}

int pa_profile_start(pa_plan* p, int max_runs) {
  if (!p) { set_err("pa_profile_start: NULL plan"); return PA_ERR_INVALID; }
  if (max_runs < 1 || max_runs > 4096) {
    set_err("pa_profile_start: max_runs %d outside [1, 4096]", max_runs);
    return PA_ERR_INVALID;
  }
  if (p->prof_cap < max_runs) {
    free_profile_events(p);
    p->prof_ev = new cudaEvent_t[2 * max_runs];
    for (int i = 0; i < 2 * max_runs; ++i) {
      cudaError_t e = cudaEventCreate(&p->prof_ev[i]);
      if (e != cudaSuccess) {
        for (int k = 0; k < i; ++k) cudaEventDestroy(p->prof_ev[k]);
        delete[] p->prof_ev;
        p->prof_ev = nullptr;
        set_err("pa_profile_start: cudaEventCreate failed: %s", cudaGetErrorString(e));
        return PA_ERR_CUDA;
      }
    }
    p->prof_cap = max_runs;
  }
  p->prof_n = 0;
  p->prof_on = 1;
  return PA_OK;
}

int pa_profile_read(pa_plan* p, float* attn_ms, int* n_runs, int* launches_per_run) {
  if (!p || !attn_ms || !n_runs) { set_err("pa_profile_read: NULL argument"); return PA_ERR_INVALID; }
  float total = 0.f;
  for (int i = 0; i < p->prof_n; ++i) {
    cudaError_t e = cudaEventSynchronize(p->prof_ev[2 * i + 1]);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, p->prof_ev[2 * i], p->prof_ev[2 * i + 1]);
    if (e != cudaSuccess) {
      set_err("pa_profile_read: %s", cudaGetErrorString(e));
      return PA_ERR_CUDA;
    }
    total += ms;
  }
  *attn_ms = total;
  *n_runs = p->prof_n;
  if (launches_per_run)
    *launches_per_run = p->last_launches;
  p->prof_on = 0;
  p->prof_n = 0;
  return PA_OK;
}


// ---------------------------------------------------------------------------
// pa_run_noalloc: the attention pass without any device allocation, for
// callers that cannot call cudaMalloc (see include/pa.h).  Its scratch is the
// file-scope array below.  Host code must not use the array's name as a
// device address (it is a host-side stand-in): the device address comes from
// cudaGetSymbolAddress, resolved once per device with that device current.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

namespace {

struct NoallocDevice {
  std::atomic<int> ready{0};
  void* scratch = nullptr;
  int n_sm = 0;
};
constexpr int kMaxDevices = 64;
NoallocDevice g_noalloc_dev[kMaxDevices];
std::mutex g_noalloc_mu;

// One-time set-up of the current device; returns PA_OK or an error code.
int noalloc_setup(int dev, NoallocDevice** out) {
  if (dev < 0 || dev >= kMaxDevices) {
    set_err("pa_run_noalloc: device %d out of range", dev);
    return PA_ERR_INVALID;
  }
  NoallocDevice& d = g_noalloc_dev[dev];
  if (!d.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!d.ready.load(std::memory_order_relaxed)) {
      int major = 0, n_sm = 0;
      cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) {
        set_err("pa_run_noalloc: device query failed: %s", cudaGetErrorString(e));
        return PA_ERR_CUDA;
      }
      if (major != 10) {
        set_err("pa_run_noalloc: device %d is not sm_100", dev);
        return PA_ERR_UNSUPPORTED;
      }
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess || ptr == nullptr) {
        set_err("pa_run_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        return PA_ERR_CUDA;
      }
      e = set_smem_attr<64>();
      if (e == cudaSuccess) e = set_smem_attr<128>();
      if (e == cudaSuccess) e = set_smem_attr<256>();
      if (e != cudaSuccess) {
        set_err("pa_run_noalloc: cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
        return PA_ERR_CUDA;
      }
      d.scratch = ptr;
      d.n_sm = n_sm;
      d.ready.store(1, std::memory_order_release);
    }
  }
  *out = &d;
  return PA_OK;
}

}  // namespace

int pa_noalloc_get_status(pa_stream_t stream, uint32_t* status, int clear) {
  if (!status) { set_err("pa_noalloc_get_status: NULL status"); return PA_ERR_INVALID; }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_err("pa_noalloc_get_status: no current CUDA device");
    return PA_ERR_CUDA;
  }
  NoallocDevice* nd = nullptr;
  int rc = noalloc_setup(dev, &nd);
  if (rc) return rc;
  pa::WsHeader* hdr = static_cast<pa::WsHeader*>(nd->scratch);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess)
    e = cudaMemcpy(status, &hdr->status, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && clear) e = cudaMemset(&hdr->status, 0, sizeof(uint32_t));
  if (e != cudaSuccess) {
    set_err("pa_noalloc_get_status: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

int pa_run_noalloc(int batch, int heads_q, int heads_kv, int head_dim, int page_size,
                   int capacity, int num_pages, float scale, const void* q, const void* k_pool,
                   const void* v_pool, const int32_t* page_table, const int32_t* seq_lens,
                   const int32_t* cu_q_lens, void* out, float* lse, pa_stream_t stream) {
  g_err[0] = 0;
  // geometry: the same envelope as pa_create_plan
  if (batch <= 0 || heads_q <= 0 || heads_kv <= 0 || head_dim <= 0 || page_size <= 0 ||
      capacity <= 0 || num_pages < 0) {
    set_err("pa_run_noalloc: batch, heads, head_dim, page_size and capacity must be > 0 "
            "and num_pages >= 0");
    return PA_ERR_INVALID;
  }
  if ((head_dim != 64 && head_dim != 128 && head_dim != 256) ||
      (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128) ||
      heads_q % heads_kv != 0 || heads_q / heads_kv > 32) {
    set_err("pa_run_noalloc: unsupported geometry (head_dim %d, page_size %d, heads %d/%d)",
            head_dim, page_size, heads_q, heads_kv);
    return PA_ERR_UNSUPPORTED;
  }
  if (!(scale >= 0.f) || !std::isfinite(scale)) {
    set_err("pa_run_noalloc: scale must be finite and >= 0 (0 = 1/sqrt(head_dim))");
    return PA_ERR_INVALID;
  }
  const int G = heads_q / heads_kv;
  const int tpb = pa::kBM / G;
  const int BN = kv_tile(head_dim);
  const long blocks_per_req = ((long)capacity * page_size + tpb - 1) / tpb;
  const long max_items = (long)batch * heads_kv * blocks_per_req;
  const size_t o_req = align_up(sizeof(pa::WsHeader), 256);
  const size_t o_aux = align_up(o_req + sizeof(int4) * (size_t)batch, 256);
  const size_t o_uoff = align_up(o_aux + sizeof(int4) * (size_t)batch, 256);
  const size_t o_split = align_up(o_uoff + sizeof(int) * (size_t)(batch + 1), 256);
  const size_t o_uoff2 = align_up(o_split + sizeof(int) * (size_t)batch, 256);
  const size_t o_items = align_up(o_uoff2 + sizeof(int) * (size_t)(batch + 1), 256);
  const size_t need = o_items + sizeof(pa::PackedItem) * (size_t)max_items;
  if (max_items > (1L << 30) || need > (size_t)PA_NOALLOC_SCRATCH_BYTES) {
    set_err("pa_run_noalloc: this geometry needs %zu bytes of scratch (%ld work items); the "
            "static scratch holds %u bytes -- use pa_create_plan / pa_run instead",
            need, max_items, (unsigned)PA_NOALLOC_SCRATCH_BYTES);
    return PA_ERR_UNSUPPORTED;
  }
  if (!q || !k_pool || !v_pool || !page_table || !seq_lens || !out) {
    set_err("pa_run_noalloc: NULL pointer (q, k_pool, v_pool, page_table, seq_lens and out "
            "are required)");
    return PA_ERR_INVALID;
  }
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out) ||
      !aligned16(page_table) || !aligned16(seq_lens) || (cu_q_lens && !aligned16(cu_q_lens)) ||
      (lse && !aligned16(lse))) {
    set_err("pa_run_noalloc: every pointer must be 16-byte aligned");
    return PA_ERR_INVALID;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_err("pa_run_noalloc: no current CUDA device");
    return PA_ERR_CUDA;
  }
  NoallocDevice* nd = nullptr;
  int rc = noalloc_setup(dev, &nd);
  if (rc) return rc;

  // tensor maps for this call, on the host stack
  const int box_h = page_size < BN ? page_size : BN;
  CUtensorMap tm_q, tm_k, tm_v;
  {
    const cuuint64_t e = 2;
    cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)heads_q,
                          (cuuint64_t)batch * capacity * page_size};
    cuuint64_t str[2] = {(cuuint64_t)head_dim * e, (cuuint64_t)heads_q * head_dim * e};
    cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)tpb};
    rc = encode(&tm_q, q, 3, dims, str, box, "q");
    if (rc) return rc;
    cuuint64_t P = num_pages > 0 ? (cuuint64_t)num_pages : (cuuint64_t)0x7fffffff;
    cuuint64_t kd[4] = {(cuuint64_t)head_dim, (cuuint64_t)heads_kv, (cuuint64_t)page_size, P};
    cuuint64_t ks[3] = {(cuuint64_t)head_dim * e, (cuuint64_t)heads_kv * head_dim * e,
                        (cuuint64_t)page_size * heads_kv * head_dim * e};
    cuuint32_t kb[4] = {64, 1, (cuuint32_t)box_h, 1};
    rc = encode(&tm_k, k_pool, 4, kd, ks, kb, "k_pool");
    if (rc) return rc;
    rc = encode(&tm_v, v_pool, 4, kd, ks, kb, "v_pool");
    if (rc) return rc;
  }

  char* base = static_cast<char*>(nd->scratch);
  pa::WsHeader* hdr = reinterpret_cast<pa::WsHeader*>(base);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the previous call's header must not leak into this one
  cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(pa::WsHeader), st);
  if (e != cudaSuccess) {
    set_err("pa_run_noalloc: cudaMemsetAsync failed: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }

  pa::SchedParams sp = {};
  sp.seq_lens = seq_lens;
  sp.cu_q_lens = cu_q_lens;
  sp.items = reinterpret_cast<pa::PackedItem*>(base + o_items);
  sp.split_list = reinterpret_cast<int*>(base + o_split);
  sp.items2 = nullptr;      // every request on the one-stage kernel
  sp.unit_off2 = reinterpret_cast<int*>(base + o_uoff2);
  sp.max_items2 = 0;
  sp.req_info = reinterpret_cast<int4*>(base + o_req);
  sp.req_aux = reinterpret_cast<int4*>(base + o_aux);
  sp.unit_off = reinterpret_cast<int*>(base + o_uoff);
  sp.hdr = hdr;
  sp.status = &hdr->status;
  sp.max_items = (int)max_items;
  sp.B = batch; sp.Hkv = heads_kv; sp.G = G; sp.C = capacity; sp.ps = page_size; sp.BN = BN;
  sp.tpb = tpb;
  sp.causal = 1;
  sp.split_cnt = nullptr;
  sp.S_max = 1;             // no KV splits on this path
  sp.forced_splits = 0;
  sp.n_ctas = attn_grid(head_dim, nd->n_sm);
  pa::pa_schedule_kernel<<<1, pa::kCostBuckets, 0, st>>>(sp);

  pa::AttnParams ap = {};
  ap.q = static_cast<const uint16_t*>(q);
  ap.page_table = page_table;
  ap.cu_q_lens = cu_q_lens;
  ap.out = static_cast<uint16_t*>(out);
  ap.lse = lse;
  ap.items = sp.items;
  ap.hdr = hdr;
  ap.part_o = nullptr;
  ap.part_lse = nullptr;
  ap.status = &hdr->status;
  ap.B = batch; ap.Hq = heads_q; ap.Hkv = heads_kv; ap.G = G; ap.C = capacity; ap.ps = page_size;
  ap.num_pages = num_pages;
  ap.S_max = 1;
  ap.tpb = tpb;
  ap.box_h = box_h;
  ap.ps_log2 = __builtin_ctz((unsigned)page_size);
  ap.box_log2 = __builtin_ctz((unsigned)box_h);
  ap.v_scale = 1.0f;
  ap.tstride = capacity;
  ap.causal = 1;
  ap.split_cnt = nullptr;
  ap.fused_merge = 0;
  ap.o_tma = 0;   // no map of out here: every block stores O directly
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)head_dim);
  ap.scale_log2 = sc * 1.4426950408889634f;
  CUtensorMap tm_none;
  memset(&tm_none, 0, sizeof(tm_none));
  e = launch_attention_d(head_dim, false, nd->n_sm, st, tm_q, tm_k, tm_v, tm_none, ap);
  if (e != cudaSuccess) {
    set_err("pa_run_noalloc: launch failed: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_err("pa_run_noalloc: launch failed: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

}  // extern "C"
