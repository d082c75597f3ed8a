// pa_kernels.cuh -- device kernels of the paged-KV GQA attention engine (sm_100a).
//
// Three kernels run per pa_run, in stream order:
//   1. pa_schedule_kernel: reads seq_lens / cu_q_lens on the device and writes
//      a work list (one item per (request, KV head, 128-row query block, KV
//      split)), longest first, plus per-request split counts.
//   2. pa_attention_kernel<D>: persistent (two CTAs per SM for D <= 128), warp-specialised:
//        warps 0-3  softmax / correction / epilogue (one thread per query row)
//        warps 4, 7 producers: page-table-driven TMA gathers of K and V pages
//                   (alternate loads: one issuing warp cannot keep HBM busy)
//        warp  5    MMA issuer: tcgen05 S = Q K^T and O += P V, TMEM accumulators
//        warp  6    Q loader: Q tiles by TMA (or plain loads for partial blocks)
//   3. pa_merge_kernel: log-sum-exp merge of split-KV partial states.
// Kernels 2 and 3 are launched as programmatic dependents of the kernel
// before them: their prologues overlap it, and `griddepcontrol.wait` orders
// their first read of its results.
//
// Sources: page-table contract and page-pool bound from "integrate PrimTS FMHA
// kernels" (TensorRT-LLM PR #17399, "Unified page-table metadata"); GQA
// packing of query heads along M, varlen queries and the mask by select from
// "Unified Triton kernel that doesn't distinguish between prefill + decode"
// (vLLM PR #16828); 128-row query tiles and split-KV decode with num_splits
// (0 = automatic) from "[Perf][FA4] Warm up dense (paged) FA4 attention
// kernels" (vLLM PR #48156, review thread on q_stage and is_split_kv).
#pragma once

#include <cstdint>
#include <cuda.h>

#include "sm100.cuh"

namespace pa {

// One unit of attention work.  Rows of the query block are packed token-major:
// row r <-> (token q_tok0 + r / G, query head kvh * G + r % G).
struct WorkItem {
  int b, kvh, split, n_splits;
  int q_tok0, n_tok;     // query tokens of the block (local to the request)
  int kv_lo, kv_hi;      // keys [kv_lo, kv_hi) processed by this item
  int kv_len, q_len;     // request lengths after validation
  int t_base;            // cu_q_lens[b]
};

// In memory an item is 32 bytes (two int4, written and read as vectors):
//   {b, kvh | split << 16 | n_splits << 24, q_tok0, t_base}
//   {kv_lo, kv_hi, kv_len, q_len}
// n_tok is min(128 / G, q_len - q_tok0).
struct __align__(16) PackedItem {
  int4 a, c;
};
static_assert(sizeof(PackedItem) == 32, "work item layout");

__device__ __forceinline__ WorkItem unpack_raw(const int4& a, const int4& c, int tpb) {
  WorkItem w;
  w.b = a.x;
  w.kvh = a.y & 0xffff;
  w.split = (a.y >> 16) & 0xff;
  w.n_splits = (a.y >> 24) & 0xff;
  w.q_tok0 = a.z;
  w.t_base = a.w;
  w.kv_lo = c.x;
  w.kv_hi = c.y;
  w.kv_len = c.z;
  w.q_len = c.w;
  w.n_tok = min(tpb, w.q_len - w.q_tok0);
  return w;
}

// The items of this CTA (blockIdx.x, + gridDim.x, ...), each read one item
// ahead so that its load latency hides behind the current item.
struct ItemStream {
  const PackedItem* items;
  int n_items, tpb, it;
  int4 na, nc;
  __device__ __forceinline__ ItemStream(const PackedItem* items_, int n, int tpb_)
      : items(items_), n_items(n), tpb(tpb_), it(blockIdx.x) {
    // plain loads: the list was written by the kernel just before this one
    if (it < n_items) { na = items[it].a; nc = items[it].c; }
  }
  __device__ __forceinline__ bool next(WorkItem& w) {
    if (it >= n_items) return false;
    w = unpack_raw(na, nc, tpb);
    it += gridDim.x;
    if (it < n_items) { na = items[it].a; nc = items[it].c; }
    return true;
  }
  __device__ __forceinline__ bool peek(WorkItem& w) const {
    if (it >= n_items) return false;
    w = unpack_raw(na, nc, tpb);
    return true;
  }
};

// Device status bits (mirror of PA_STATUS_* in pa.h).
constexpr unsigned kStatusBadPage = 1u << 0;
constexpr unsigned kStatusQgtKv = 1u << 1;
constexpr unsigned kStatusKvGtCap = 1u << 2;
constexpr unsigned kStatusBadCuQ = 1u << 3;
constexpr unsigned kStatusTimeout = 1u << 4;

struct WsHeader {
  unsigned status;
  int n_items;
  int n_split_reqs;   // requests split over KV (entries of the split list)
  int n_items2;       // items of the second list (query-block pairs, or widened requests)
  int n_wide_pages;   // pages of the widened requests (E4M3 pools, second list)
  int n_items_b;      // one-token segment after the main list's n_items (split_decode)
  int pad[58];
};

constexpr int kBM = 128;              // query rows per tile (tcgen05 M)
constexpr int kThreads = 256;         // 8 warps
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kQWarp = 6;
constexpr int kProducer2Warp = 7;     // second K/V producer: one issuing warp per CTA
                                      // cannot keep HBM busy with page-sized boxes
constexpr int kCostBuckets = 1024;
constexpr int kSchedSmemReqs = 3072;  // unit offsets of up to this many requests live in smem
constexpr int kMaxSplits = 64;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows > 2^8
// Compensated P * V.  The softmax weights feed the P V product as 16-bit
// values; rounding them costs up to 2^-9 of sum_j P_j |V_j| per row.  With
// many keys these errors average out, but a row that sees only a few keys
// can have |O| of 2 to 4, where this error plus the final bf16 rounding of O
// (up to 2^-8 |O|) can pass 1e-2.  Items holding a row that sees fewer than
// kCompKeys keys in total therefore also multiply the rounding remainder
// P_lo = 16-bit(P - P_hi) by V into the same accumulator (P_hi + P_lo
// carries P to about 2^-17), leaving only the final rounding of O.  Only the
// first query blocks of each request qualify, so the extra products are a
// small fraction of the work.
constexpr int kCompKeys = 64;

// Tile configuration per head dimension.  D = 64 and 128 run two CTAs per SM
// (64-key tiles, 256 TMEM columns, ~100 KB of shared memory each): two
// independent load -> S -> softmax -> P V chains per SM hide each other's
// latencies, which one CTA per SM cannot.  D = 256 needs the whole SM.
// F8: E4M3 pools.  The producers' TMA boxes land in NST fp8 staging tiles and
// the widening warp(s) turn them into fp16 in the 16-bit slots the MMAs read.
// The loads in flight are what hides HBM latency, so F8 trades 16-bit slots
// for staging tiles in the same shared memory: four staging tiles, and two
// slots for D = 128 or three for D = 256 (the widening is quick next to a load;
// two staging tiles with four or three slots was 7 % / 5 % slower).
template <int D, bool F8 = false>
struct TileCfg {
  static_assert(!F8 || D >= 128, "E4M3 pools: head_dim 128 or 256");
  static constexpr int CTAS = (D == 256) ? 1 : 2;      // CTAs per SM
  // E4M3 widening warps.  D = 256 (one CTA per SM): a warpgroup of four that
  // shares every tile (one warp widened ~8 codes per clock, a third of the
  // HBM rate), with a second producer; D = 128 (two CTAs per SM, every
  // register taken): one.
  static constexpr int NCONV = (F8 && D == 256) ? 4 : 1;
  static constexpr int THREADS = (NCONV > 1) ? 384 : 256;
  // two CTAs: 16 warps on 4 sub-partitions, 4 warps x 32 lanes x 128 = 16 K
  // registers each; 384 threads: 168 (65 536 / 384, rounded down to 8)
  static constexpr int MAXREG = (CTAS == 2) ? 128 : (THREADS == 384 ? 168 : 255);
  static constexpr int BN = 64;                       // keys per KV tile
  static constexpr int DCH = D / 64;                  // 128-byte column chunks per row
  static constexpr int Q_CHUNK = kBM * 128;           // bytes of one Q column chunk
  static constexpr int Q_BYTES = kBM * D * 2;
  static constexpr int SLOT_CHUNK = BN * 128;         // bytes of one K/V column chunk
  static constexpr int SLOT_BYTES = BN * D * 2;
  static constexpr int QBUF = (D == 64) ? 2 : 1;      // Q tiles in flight
  static constexpr int NSLOT = F8 ? (D == 128 ? 2 : 3) : ((D == 64) ? 8 : (D == 128 ? 4 : 5));
  static constexpr int NST = F8 ? 4 : 0;              // fp8 staging tiles
  static constexpr int STAGE_BYTES = BN * D;          // D / 128 chunks of BN rows x 128 bytes
  static constexpr int O_COL = 2 * BN;                // TMEM: S0 [0,BN), S1 [BN,2BN), O
  static constexpr int TMEM_COLS = (O_COL + D <= 256) ? 256 : 512;
  static constexpr int OCH = (CTAS == 2) ? 1 : 2;     // 32-column O chunks per TMEM wait
  // barriers: q_full[QBUF], q_empty[QBUF], kv_full[NSLOT], kv_empty[NSLOT], s_full[2],
  //           p_full[2], pv_done[2], o_empty, drain, st_full[NST], st_empty[NST],
  //           merge (the softmax warps' fused split-merge hand-shake)
  static constexpr int B_QFULL = 0, B_QEMPTY = QBUF, B_KVFULL = 2 * QBUF,
                       B_KVEMPTY = 2 * QBUF + NSLOT, B_SFULL = 2 * QBUF + 2 * NSLOT,
                       B_PFULL = B_SFULL + 2, B_PVDONE = B_PFULL + 2, B_OEMPTY = B_PVDONE + 2,
                       B_DRAIN = B_OEMPTY + 1, B_STFULL = B_DRAIN + 1,
                       B_STEMPTY = B_STFULL + NST, B_MERGE = B_STEMPTY + NST,
                       NBAR = B_MERGE + 1;
  static constexpr int BAR_BYTES = 512;
  // epilogue staging: per softmax warp 32 rows x 32 columns of bf16 (64-byte
  // swizzle); D = 256 has no room for it next to its K/V slots
  static constexpr int EPI_WARP_BYTES = 32 * 64;
  static constexpr int EPI_BYTES = (D == 256) ? 0 : 4 * EPI_WARP_BYTES;
  static constexpr int SMEM_BYTES = 1024 + QBUF * Q_BYTES + NSLOT * SLOT_BYTES +
                                    NST * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
  static_assert(NBAR * 8 + 16 <= BAR_BYTES, "barrier area");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(CTAS == 1 || 2 * (SMEM_BYTES + 1024) <= 228 * 1024, "two CTAs per SM");
  static_assert(O_COL + D <= TMEM_COLS, "TMEM columns");
};

struct AttnParams {
  const uint16_t* q;          // bf16 [T, Hq, D]
  const int* page_table;      // [B, C]
  const int* cu_q_lens;       // [B+1] or nullptr
  uint16_t* out;              // bf16 [T, Hq, D]
  float* lse;                 // [T, Hq] or nullptr
  const PackedItem* items;
  const WsHeader* hdr;
  float* part_o;              // [B*Hkv*S_max*128, D]
  float* part_lse;            // [B*Hkv*S_max*128]
  unsigned* status;
  int B, Hq, Hkv, G, C, ps, num_pages, S_max, tpb, box_h;
  int ps_log2, box_log2;      // log2 of ps and box_h (both powers of two)
  int tstride;                // page-table row stride (>= C)
  int causal;                 // 1: causal mask aligned to the end of KV; 0: all keys
  int o_tma;                  // 1: full blocks store O through the tensor map of out
  int* split_cnt;             // [B * Hkv] arrivals of split softmax warps (zeroed per run)
  int fused_merge;            // 1: the last split warp of a (request, KV head) merges
  float scale_log2;           // softmax scale * log2(e) (times the K descale for E4M3 pools)
  float v_scale;              // V descale of E4M3 pools (1 for bf16 pools)
  int list;                   // 0: the main list; 1: items is the second list (hdr->n_items2);
                              // 2: the one-token segment after the main list (hdr->n_items_b)
};

// The work list a kernel walks (see AttnParams::list).
__device__ __forceinline__ const PackedItem* list_items(const AttnParams& p) {
  return p.list == 2 ? p.items + p.hdr->n_items : p.items;
}
__device__ __forceinline__ int list_count(const AttnParams& p) {
  return p.list == 1 ? p.hdr->n_items2 : (p.list == 2 ? p.hdr->n_items_b : p.hdr->n_items);
}

constexpr int kSoftmaxWarps = 4;      // softmax warps per CTA in every attention kernel

// Merge of one row's split states by one warp: L = ln sum_s exp(L_s),
// O = sum_s exp(L_s - L) O_s, the exact identity for attention states over
// disjoint key ranges; empty splits (L_s = -inf) have weight 0.  Partials are
// read through L2 (ld.global.cg): in the fused path other CTAs wrote them
// during this launch.  part rows of the split s are base + s * 128.
__device__ __forceinline__ void merge_one_row(const float* part_o, const float* part_lse,
                                              size_t base, int ns, int D, uint16_t* out_row,
                                              float* lse_out) {
  const int lane = threadIdx.x & 31;
  const float l0 = lane < ns ? __ldcg(part_lse + base + (size_t)lane * kBM) : -INFINITY;
  const float l1 = lane + 32 < ns ? __ldcg(part_lse + base + (size_t)(lane + 32) * kBM) : -INFINITY;
  float m = fmaxf(l0, l1);
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float e = 0.f;
  if (m != -INFINITY)
    e = (l0 == -INFINITY ? 0.f : expf(l0 - m)) + (l1 == -INFINITY ? 0.f : expf(l1 - m));
  for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
  const float L = (m == -INFINITY) ? -INFINITY : m + logf(e);
  const float w0 = (L == -INFINITY || l0 == -INFINITY) ? 0.f : expf(l0 - L);
  const float w1 = (L == -INFINITY || l1 == -INFINITY) ? 0.f : expf(l1 - L);
  // lane owns columns 4 lane .. 4 lane + 3 of each 128-wide chunk (D <= 256:
  // at most two chunks); both chunks of a split are loaded in the same pass,
  // eight splits per unrolled step, so up to 16 loads per lane are in flight
  const int d_a = lane * 4, d_b = 128 + lane * 4;
  const bool act_a = d_a < D, act_b = d_b < D;
  float4 acc_a = make_float4(0.f, 0.f, 0.f, 0.f), acc_b = acc_a;
#pragma unroll 8
  for (int s = 0; s < ns; ++s) {
    const float wgt = __shfl_sync(0xffffffffu, s < 32 ? w0 : w1, s & 31);
    const float* row = part_o + (base + (size_t)s * kBM) * D;
    if (act_a) {
      const float4 o = __ldcg(reinterpret_cast<const float4*>(row + d_a));
      acc_a.x = fmaf(wgt, o.x, acc_a.x);
      acc_a.y = fmaf(wgt, o.y, acc_a.y);
      acc_a.z = fmaf(wgt, o.z, acc_a.z);
      acc_a.w = fmaf(wgt, o.w, acc_a.w);
    }
    if (act_b) {
      const float4 o = __ldcg(reinterpret_cast<const float4*>(row + d_b));
      acc_b.x = fmaf(wgt, o.x, acc_b.x);
      acc_b.y = fmaf(wgt, o.y, acc_b.y);
      acc_b.z = fmaf(wgt, o.z, acc_b.z);
      acc_b.w = fmaf(wgt, o.w, acc_b.w);
    }
  }
  if (act_a) {
    uint2 pk;
    pk.x = pack_bf16x2(acc_a.x, acc_a.y);
    pk.y = pack_bf16x2(acc_a.z, acc_a.w);
    *reinterpret_cast<uint2*>(out_row + d_a) = pk;
  }
  if (act_b) {
    uint2 pk;
    pk.x = pack_bf16x2(acc_b.x, acc_b.y);
    pk.y = pack_bf16x2(acc_b.z, acc_b.w);
    *reinterpret_cast<uint2*>(out_row + d_b) = pk;
  }
  if (lane == 0 && lse_out) *lse_out = L;
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort);

// Fused split-KV reduction.  Called by all four softmax warps of a CTA after
// they wrote their share of a split item's partials (or nothing, for rows they
// do not own).  The CTA, not the warp, counts itself in the (request, KV head)
// counter: every warp publishes its writes (__threadfence) and arrives on the
// CTA's merge barrier `mbar` (count 4); once all four have, warp 0 takes a
// ticket and tells the others through `flag` (a second phase of the same
// barrier) whether this CTA brought the count to n_splits.  If so, every
// split's partials are visible and the four warps merge the item's rows
// between them (row r by warp r % 4).  Each call uses two phases of the
// barrier (parities 0 and 1); the waits are bounded, so a warp that gave up
// elsewhere cannot hang the others.  No CTA waits for another CTA.
__device__ __forceinline__ void split_arrive_and_merge(const AttnParams& p, const WorkItem& w,
                                                       int D, uint32_t mbar, volatile int* flag,
                                                       volatile int* abort) {
  const int warp = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31;
  __threadfence();
  __syncwarp();
  if (lane == 0) mbar_arrive(mbar);
  if (!warp_wait(mbar, 0, abort)) return;
  if (warp == 0 && lane == 0)
    *flag = atomicAdd(p.split_cnt + (size_t)w.b * p.Hkv + w.kvh, 1) == w.n_splits - 1;
  __syncwarp();
  if (lane == 0) mbar_arrive(mbar);
  if (!warp_wait(mbar, 1, abort)) return;
  if (!*flag) return;
  __threadfence();
  const int n_rows = w.n_tok * p.G;
  for (int r = warp; r < n_rows; r += kSoftmaxWarps) {
    const size_t base = ((size_t)w.b * p.Hkv + w.kvh) * p.S_max * kBM + r;
    const size_t orow = (size_t)(w.t_base + w.q_tok0 + r / p.G) * p.Hq + w.kvh * p.G + r % p.G;
    merge_one_row(p.part_o, p.part_lse, base, w.n_splits, D, p.out + orow * D,
                  p.lse ? p.lse + orow : nullptr);
  }
}

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Does item w hold a row that sees fewer than kCompKeys keys (all of its keys
// from key 0, whatever the item's own key range)?  The row with the fewest is
// the item's first query row: causal limit kv_len - q_len + q_tok0 + 1.
__device__ __forceinline__ bool item_compensated(const WorkItem& w, int causal) {
  const int vis0 = causal ? min(w.kv_len, w.kv_len - w.q_len + w.q_tok0 + 1) : w.kv_len;
  return vis0 < kCompKeys;
}

__device__ __forceinline__ int item_tiles(const WorkItem& w, int BN) {
  return w.kv_hi > w.kv_lo ? ceil_div(w.kv_hi - w.kv_lo, BN) : 0;
}

// Order in which K and V tiles of an item are loaded and consumed:
// K0, K1, V0, K2, V1, ..., K(n-1), V(n-2), V(n-1).  S for tile j+1 is issued
// before P*V of tile j so the tensor core works while softmax runs.
__device__ __forceinline__ void kv_sequence(int s, int n, int& j, bool& is_v) {
  if (s == 0) { j = 0; is_v = false; }
  else if (s == 2 * n - 1) { j = n - 1; is_v = true; }
  else if (s & 1) { j = (s + 1) >> 1; is_v = false; }
  else { j = (s >> 1) - 1; is_v = true; }
}

// mbar_wait executed by every lane of a warp, with a warp-uniform result: a
// lane that gives up makes the whole warp give up, so no lane is left behind
// at a later warp-collective instruction.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

// Wait without the abort shortcut, for draining in-flight copies at exit.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 100000000ull) return;  // 100 ms
  }
}

// =========================================================================== scheduler
struct SchedParams {
  const int* seq_lens;
  const int* cu_q_lens;
  PackedItem* items;
  PackedItem* items2;  // second list (pairs or widened requests), or nullptr
  int* unit_off2;      // [B + 1] exclusive prefix sum of second-list units
  int max_items2;
  // E4M3 pools: requests with two or more query blocks are widened once into a
  // 16-bit scratch pool of wide_cap pages, in request order while they fit,
  // and their blocks go to the second list (one unit per block).  wide_cap = 0:
  // no widening.  wpre[b] = first scratch page of request b ([B + 1] entries,
  // non-decreasing; requests that are not widened own no pages).
  int wide_cap;
  int* wpre;
  // 1: requests of one query token form a second segment of the main list
  // (items [n_items, n_items + n_items_b)), for the decode kernel; the rest
  // stay in the first segment
  int split_decode;
  int* split_list;     // [B] requests with more than one split
  int4* req_info;      // [B] {n_splits, q_len, t_base, kv_len}
  int4* req_aux;       // [B] {units, tiles per split, KV tiles of the single block, 0}
  int* unit_off;       // [B + 1] exclusive prefix sum of units
  WsHeader* hdr;        // this run's header (n_items, n_split_reqs, n_items2)
  unsigned* status;     // the plan's status word
  int max_items;
  int B, Hkv, G, C, ps, BN, tpb, S_max, forced_splits, n_ctas;
  int causal;          // 0: every row of a request sees all of its keys
  int* split_cnt;      // [B * Hkv] fused-merge counters, zeroed here every run (or nullptr)
};

struct ReqInfo {
  int q_len, t_base, kv_len;
  unsigned flags;
};

__device__ __forceinline__ ReqInfo read_request(const SchedParams& p, int b) {
  ReqInfo r;
  r.flags = 0;
  if (p.cu_q_lens) {
    const int a = p.cu_q_lens[b], e = p.cu_q_lens[b + 1];
    if (a < 0 || e < a || (b == 0 && a != 0)) {
      r.flags |= kStatusBadCuQ;
      r.q_len = 0;
      r.t_base = a < 0 ? 0 : a;
    } else {
      r.q_len = e - a;
      r.t_base = a;
    }
  } else {
    r.q_len = 1;
    r.t_base = b;
  }
  const int cap = p.C * p.ps;
  int kv = p.seq_lens[b];
  if (kv < 0) { r.flags |= kStatusKvGtCap; kv = 0; }
  if (kv > cap) { r.flags |= kStatusKvGtCap; kv = cap; }
  r.kv_len = kv;
  if (r.q_len > kv) r.flags |= kStatusQgtKv;
  if (r.q_len > cap) r.q_len = cap;   // keeps the work list within its bound
  return r;
}

// Keys visible to the last row of query block [q0, q0 + n): the causal limit
// aligned to the end of the request's KV, clamped to [0, kv_len]; all of them
// without the causal mask.
__device__ __forceinline__ int block_kv_hi(int q_len, int kv_len, int q0, int n, int causal) {
  if (!causal) return kv_len;
  int hi = q0 + n + (kv_len - q_len);
  return hi < 0 ? 0 : (hi > kv_len ? kv_len : hi);
}

__device__ __forceinline__ int n_qblocks(int q_len, int tpb) {
  return q_len > 0 ? (q_len + tpb - 1) / tpb : 0;
}

__device__ __forceinline__ int cost_bucket(int tiles) {
  return tiles < kCostBuckets ? tiles : kCostBuckets - 1;
}

// Exclusive scan of one int per thread over a 1024-thread block; returns the
// thread's exclusive prefix and writes the block total to *total.
__device__ __forceinline__ int block_scan_1024(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const int r = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[31];
  __syncthreads();
  return r;
}

// Cost (KV tiles) and shape of unit k of request b.
struct Unit {
  int q0, n_tok, kv_lo, kv_hi, split, cost;
};

__device__ __forceinline__ Unit unit_of(const SchedParams& p, const int4& ri, const int4& ra,
                                        int k) {
  Unit u;
  const int ns = ri.x, q_len = ri.y, kv_len = ri.w;
  if (ns > 1) {
    const int per = ra.y, tiles = ra.z;
    u.q0 = 0;
    u.n_tok = q_len;
    u.split = k;
    u.kv_lo = k * per * p.BN;
    u.kv_hi = min(block_kv_hi(q_len, kv_len, 0, q_len, p.causal), (k + 1) * per * p.BN);
    u.cost = min(per, tiles - k * per);
  } else {
    u.q0 = k * p.tpb;
    u.n_tok = min(p.tpb, q_len - u.q0);
    u.split = 0;
    u.kv_lo = 0;
    u.kv_hi = block_kv_hi(q_len, kv_len, u.q0, u.n_tok, p.causal);
    u.cost = ceil_div(u.kv_hi, p.BN);
  }
  return u;
}

// One CTA of 1024 threads.
//   1. validate every request, count the KV tiles of all work;
//   2. choose splits (about four items per CTA over all work, or the forced
//      count) for requests whose packed rows fit one 128-row tile; count the
//      units (query blocks or splits) of each request and prefix-sum them;
//   3. histogram of unit costs, scanned in descending cost order;
//   4. every unit writes its Hkv items at its cost bucket's cursor, so the
//      work list comes out longest first.
// Atomics on the histogram and the cursors are aggregated per warp.
__global__ void __launch_bounds__(1024) pa_schedule_kernel(SchedParams p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // cost buckets of the main list's two segments (the second one only with
  // split_decode): [0, kCostBuckets) and [kCostBuckets, 2 kCostBuckets)
  __shared__ int hist[2 * kCostBuckets];
  __shared__ int cursor[2 * kCostBuckets];
  __shared__ unsigned long long total_tiles;
  __shared__ int s_chunk;
  __shared__ unsigned s_flags;
  __shared__ int warp_sums[32];
  const int tid = threadIdx.x, lane = tid & 31;
  for (int i = tid; i < 2 * kCostBuckets; i += blockDim.x) hist[i] = 0;
  if (tid == 0) { total_tiles = 0; s_flags = 0; }
  if (p.split_cnt)
    for (int i = tid; i < p.B * p.Hkv; i += blockDim.x) p.split_cnt[i] = 0;
  __syncthreads();

  // 1.
  unsigned long long my_tiles = 0;
  unsigned my_flags = 0;
  for (int b = tid; b < p.B; b += blockDim.x) {
    const ReqInfo r = read_request(p, b);
    my_flags |= r.flags;
    const int nb = n_qblocks(r.q_len, p.tpb);
    int t = 0;
    for (int m = 0; m < nb; ++m) {
      const int q0 = m * p.tpb;
      t += ceil_div(block_kv_hi(r.q_len, r.kv_len, q0, min(p.tpb, r.q_len - q0), p.causal), p.BN);
    }
    my_tiles += (unsigned long long)p.Hkv * t;
  }
  for (int o = 16; o > 0; o >>= 1) {
    my_tiles += __shfl_xor_sync(0xffffffffu, my_tiles, o);
    my_flags |= __shfl_xor_sync(0xffffffffu, my_flags, o);
  }
  if (lane == 0) {
    atomicAdd(&total_tiles, my_tiles);
    if (my_flags) atomicOr(&s_flags, my_flags);
  }
  __syncthreads();
  if (tid == 0) {
    // about four items per CTA: with the longest-first order that balances
    // uneven requests without making the split merge too long
    const unsigned long long target = (unsigned long long)p.n_ctas * 4ull;
    const unsigned long long c = (total_tiles + target - 1) / target;
    s_chunk = (int)(c < 4 ? 4 : (c > (1ull << 30) ? (1ull << 30) : c));
    if (s_flags) atomicOr(p.status, s_flags);
  }
  __syncthreads();
  const int chunk = s_chunk;

  // 2.  A request with two or more query blocks goes to the second list when
  // items2 != nullptr: with the two-stage prefill kernel one unit per pair of
  // consecutive blocks; with E4M3 pools (wide_cap > 0) one unit per block, if
  // its pages still fit the scratch pool (the request is then widened once
  // and read as 16-bit tiles).  Every other request goes to the main list.
  __shared__ int s_nsplit;
  __shared__ int s_wide_pages;
  __shared__ int s_uoff[kSchedSmemReqs + 1];
  __shared__ int s_uoff2[kSchedSmemReqs + 1];
  if (tid == 0) { s_nsplit = 0; s_wide_pages = 0; }
  __syncthreads();
  const bool wide_mode = p.items2 != nullptr && p.wide_cap > 0;
  int running = 0, running2 = 0, running_pg = 0;
  for (int b0 = 0; b0 < p.B; b0 += blockDim.x) {
    const int b = b0 + tid;
    int units = 0, units2 = 0, pages = 0, nb = 0;
    ReqInfo r = {0, 0, 0, 0u};
    if (b < p.B) {
      r = read_request(p, b);
      nb = n_qblocks(r.q_len, p.tpb);
      if (wide_mode && nb >= 2) pages = ceil_div(r.kv_len, p.ps);
    }
    // scratch pages: the candidates' exclusive prefix, in request order
    int total_pg;
    const int pg0 = running_pg + block_scan_1024(pages, warp_sums, &total_pg);
    const bool wide = pages > 0 && pg0 + pages <= p.wide_cap;
    if (b < p.B) {
      const int tiles = ceil_div(block_kv_hi(r.q_len, r.kv_len, 0, r.q_len, p.causal), p.BN);
      int ns = 1, per = tiles > 0 ? tiles : 1;
      if (nb == 1 && p.S_max > 1 && tiles > 1) {
        int sp = p.forced_splits > 0 ? p.forced_splits : ceil_div(tiles, chunk);
        sp = min(sp, min(p.S_max, tiles));
        if (sp < 1) sp = 1;
        per = ceil_div(tiles, sp);
        ns = ceil_div(tiles, per);
      }
      if (wide) units2 = nb;
      else if (!wide_mode && p.items2 != nullptr && ns == 1 && nb >= 2) units2 = (nb + 1) / 2;
      else units = ns > 1 ? ns : nb;
      p.req_info[b] = make_int4(ns, r.q_len, r.t_base, r.kv_len);
      p.req_aux[b] = make_int4(units, per, tiles, 0);
      if (ns > 1) p.split_list[atomicAdd(&s_nsplit, 1)] = b;
      if (wide_mode) p.wpre[b] = pg0;
      if (wide) atomicMax(&s_wide_pages, pg0 + pages);
    }
    running_pg += total_pg;
    int total, total2;
    const int off = block_scan_1024(units, warp_sums, &total);
    const int off2 = block_scan_1024(units2, warp_sums, &total2);
    if (b < p.B) {
      p.unit_off[b] = running + off;
      p.unit_off2[b] = running2 + off2;
      if (b < kSchedSmemReqs) {
        s_uoff[b] = running + off;
        s_uoff2[b] = running2 + off2;
      }
    }
    running += total;
    running2 += total2;
  }
  if (tid == 0) {
    p.unit_off[p.B] = running;
    p.unit_off2[p.B] = running2;
    if (p.B <= kSchedSmemReqs) {
      s_uoff[p.B] = running;
      s_uoff2[p.B] = running2;
    }
    p.hdr->n_split_reqs = s_nsplit;
    const int n2 = running2 * p.Hkv;
    p.hdr->n_items2 = n2 < p.max_items2 ? n2 : p.max_items2;
    p.hdr->n_wide_pages = s_wide_pages;
    if (wide_mode) p.wpre[p.B] = running_pg;
  }
  __syncthreads();
  const int U = running;
  const int* uoff = p.B <= kSchedSmemReqs ? s_uoff : p.unit_off;
  const int U2 = running2;
  const int* uoff2 = p.B <= kSchedSmemReqs ? s_uoff2 : p.unit_off2;

  // 2b.  Second list: each request's units (pairs, or single blocks of a
  // widened request) stay together, last unit (most keys) first; a unit writes
  // its Hkv items (one per KV head) at consecutive places.
  const int bpu = wide_mode ? 1 : 2;   // query blocks per unit
  for (int u0 = 0; u0 < U2; u0 += blockDim.x) {
    const int u = u0 + tid;
    if (u < U2) {
      int lo = 0, hi = p.B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (uoff2[mid] <= u) lo = mid; else hi = mid - 1;
      }
      const int b = lo;
      const int4 ri = p.req_info[b];
      const int k = u - uoff2[b];
      const int units2 = uoff2[b + 1] - uoff2[b];
      const int unit = units2 - 1 - k;
      const int q0 = bpu * unit * p.tpb;
      const int ntok = min(bpu * p.tpb, ri.y - q0);
      const int hi_kv = block_kv_hi(ri.y, ri.w, q0, ntok, p.causal);
      const int pos = u * p.Hkv;
      for (int g = 0; g < p.Hkv; ++g) {
        if (pos + g < p.max_items2) {
          PackedItem* dst = p.items2 + pos + g;
          dst->a = make_int4(b, g | (1 << 24), q0, ri.z);
          dst->c = make_int4(0, hi_kv, ri.w, ri.y);
        }
      }
    }
  }

  // 3.  Ordering.  A request with several query blocks (prefill) keeps its
  // units together, last block (most keys) first, and the block of units is
  // placed by its largest cost: the CTAs then work on few requests at a time
  // and the K/V tiles those blocks share are re-read from L2, not DRAM.  Other
  // units (decode-like, KV splits) are placed one by one, longest first.
  for (int b = tid; b < p.B; b += blockDim.x) {
    const int4 ri = p.req_info[b], ra = p.req_aux[b];
    if (ri.x == 1 && ra.x > 1) atomicAdd(&hist[cost_bucket(ra.z)], ra.x * p.Hkv);
  }
  for (int u0 = 0; u0 < U; u0 += blockDim.x) {
    const int u = u0 + tid;
    int key = -1 - lane;     // distinct per idle lane
    if (u < U) {
      int lo = 0, hi = p.B - 1;            // last b with unit_off[b] <= u
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (uoff[mid] <= u) lo = mid; else hi = mid - 1;
      }
      const int4 ri = p.req_info[lo], ra = p.req_aux[lo];
      if (!(ri.x == 1 && ra.x > 1))
        key = cost_bucket(unit_of(p, ri, ra, u - uoff[lo]).cost) +
              ((p.split_decode && ri.y == 1) ? kCostBuckets : 0);
    }
    const unsigned grp = __match_any_sync(0xffffffffu, key);
    if (key >= 0 && lane == __ffs(grp) - 1) atomicAdd(&hist[key], __popc(grp) * p.Hkv);
  }
  __syncthreads();
  {
    // each segment longest first; the one-token segment after the other
    const int bucket = kCostBuckets - 1 - tid;
    int total_a, total_b;
    const int before_a = block_scan_1024(hist[bucket], warp_sums, &total_a);
    const int before_b = block_scan_1024(hist[kCostBuckets + bucket], warp_sums, &total_b);
    cursor[bucket] = before_a;
    cursor[kCostBuckets + bucket] = total_a + before_b;
    if (tid == 0) {
      const int na = total_a < p.max_items ? total_a : p.max_items;
      const int nb = total_b < p.max_items - na ? total_b : p.max_items - na;
      p.hdr->n_items = na;
      p.hdr->n_items_b = nb;
    }
  }
  __syncthreads();
  for (int b = tid; b < p.B; b += blockDim.x) {
    const int4 ri = p.req_info[b];
    int4 ra = p.req_aux[b];
    if (ri.x == 1 && ra.x > 1) {
      ra.w = atomicAdd(&cursor[cost_bucket(ra.z)], ra.x * p.Hkv);
      p.req_aux[b] = ra;
    }
  }
  __syncthreads();

  // 4.  Each unit owns Hkv consecutive items; the warp writes the items of its
  // 32 units cooperatively (item i of the warp -> unit i / Hkv, head i % Hkv),
  // so consecutive lanes store consecutive 32-byte items.
  for (int u0 = 0; u0 < U; u0 += blockDim.x) {
    const int u = u0 + tid;
    int key = -1 - lane;
    int b = 0;
    Unit un = {0, 0, 0, 0, 0, 0};
    int4 ri = make_int4(0, 0, 0, 0);
    int pos = -1;
    if (u < U) {
      int lo = 0, hi = p.B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (uoff[mid] <= u) lo = mid; else hi = mid - 1;
      }
      b = lo;
      ri = p.req_info[b];
      const int4 ra = p.req_aux[b];
      const int k = u - uoff[b];
      un = unit_of(p, ri, ra, k);
      if (ri.x == 1 && ra.x > 1) pos = ra.w + (ra.x - 1 - k) * p.Hkv;   // grouped request
      else key = cost_bucket(un.cost) + ((p.split_decode && ri.y == 1) ? kCostBuckets : 0);
    }
    const unsigned grp = __match_any_sync(0xffffffffu, key);
    const int leader = __ffs(grp) - 1;
    int base = 0;
    if (key >= 0 && lane == leader) base = atomicAdd(&cursor[key], __popc(grp) * p.Hkv);
    base = __shfl_sync(0xffffffffu, base, leader);
    if (key >= 0) pos = base + __popc(grp & ((1u << lane) - 1)) * p.Hkv;
    const int packed = (un.split << 16) | (ri.x << 24);
    for (int i0 = 0; i0 < 32 * p.Hkv; i0 += 32) {
      const int i = i0 + lane;
      const int src = i / p.Hkv, g = i - src * p.Hkv;
      const int spos = __shfl_sync(0xffffffffu, pos, src);
      const int sb = __shfl_sync(0xffffffffu, b, src);
      const int spk = __shfl_sync(0xffffffffu, packed, src);
      const int sq0 = __shfl_sync(0xffffffffu, un.q0, src);
      const int stb = __shfl_sync(0xffffffffu, ri.z, src);
      const int slo = __shfl_sync(0xffffffffu, un.kv_lo, src);
      const int shi = __shfl_sync(0xffffffffu, un.kv_hi, src);
      const int skv = __shfl_sync(0xffffffffu, ri.w, src);
      const int sql = __shfl_sync(0xffffffffu, ri.y, src);
      if (spos >= 0 && spos + g < p.max_items) {
        PackedItem* dst = p.items + spos + g;
        dst->a = make_int4(sb, g | spk, sq0, stb);
        dst->c = make_int4(slo, shi, skv, sql);
      }
    }
  }
  // this kernel may have started while the previous run's kernels were still
  // running (it only wrote the other set of buffers); finishing only after
  // them orders every later kernel after the previous run as well
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// =========================================================================== attention
// Q loader warp: one Q tile per item, into the single Q buffer.  Full blocks
// inside [0, T) use one TMA box per 64-column chunk; partial blocks (decode,
// last block of a request) use plain 16-byte loads of the live rows only,
// stored with the same 128-byte swizzle the TMA applies (16-byte unit u of
// row r lands at unit u ^ (r % 8) of that row).  With E4M3 pools (F8) the MMAs
// run in fp16: every block takes the plain-load path and is rounded to fp16
// (magnitudes past 65504 saturate) on the way to shared memory.
template <int D, bool F8>
__device__ __forceinline__ void q_loader_role(const CUtensorMap* tm_q, const AttnParams& p,
                                              uint32_t sQ, uint32_t bar0, int n_items,
                                              volatile int* abort) {
  using C = TileCfg<D, F8>;
  const int lane = threadIdx.x & 31;
  const int G = p.G;
  const int T = p.cu_q_lens ? p.cu_q_lens[p.B] : p.B;
  uint32_t q_cnt = 0;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (items.next(w)) {
    if (item_tiles(w, C::BN) == 0) continue;
    const uint32_t qb = q_cnt % C::QBUF;
    const uint32_t sQb = sQ + qb * C::Q_BYTES;
    const uint32_t qfull = bar0 + 8 * (C::B_QFULL + qb);
    if (!warp_wait(bar0 + 8 * (C::B_QEMPTY + qb), ((q_cnt / C::QBUF) & 1) ^ 1, abort)) break;
    const int t0 = w.t_base + w.q_tok0;
    if (!F8 && w.n_tok == p.tpb && t0 + p.tpb <= T) {
      if (lane == 0) {
        mbar_arrive_expect_tx(qfull, C::DCH * p.tpb * G * 128);
        for (int c = 0; c < C::DCH; ++c)
          tma_load_3d(sQb + c * C::Q_CHUNK, tm_q, qfull, c * 64, w.kvh * G, t0);
      }
    } else {
      const int rows = w.n_tok * G;
      const int units = rows * (D / 8);
      for (int u0 = 0; u0 < units; u0 += 8 * 32) {
        uint4 v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {          // all loads first, then the stores
          const int u = u0 + k * 32 + lane;
          if (u < units) {
            const int r = u / (D / 8), c16 = u % (D / 8);
            const int t = t0 + r / G, h = w.kvh * G + r % G;
            v[k] = __ldg(reinterpret_cast<const uint4*>(p.q + ((size_t)t * p.Hq + h) * D) + c16);
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int u = u0 + k * 32 + lane;
          if (u < units) {
            const int r = u / (D / 8), c16 = u % (D / 8);
            const uint32_t dst =
                sQb + (c16 >> 3) * C::Q_CHUNK + r * 128 + (((c16 & 7) ^ (r & 7)) << 4);
            if constexpr (F8) {
              v[k].x = bf16x2_to_f16x2_sat(v[k].x);
              v[k].y = bf16x2_to_f16x2_sat(v[k].y);
              v[k].z = bf16x2_to_f16x2_sat(v[k].z);
              v[k].w = bf16x2_to_f16x2_sat(v[k].w);
            }
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[k].x),
                         "r"(v[k].y), "r"(v[k].z), "r"(v[k].w)
                         : "memory");
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(qfull);
    }
    ++q_cnt;
    // Q is read once, so it always comes from DRAM: pull the next item's Q
    // tile into L2 now so that its load is short when its turn comes.
    WorkItem nw;
    if (!F8 && lane == 0 && items.peek(nw) && item_tiles(nw, C::BN) > 0 && nw.n_tok == p.tpb) {
      const int tn = nw.t_base + nw.q_tok0;
      if (tn + p.tpb <= T)
        for (int c = 0; c < C::DCH; ++c) tma_prefetch_l2_3d(tm_q, c * 64, nw.kvh * G, tn);
    }
  }
  if (*abort && lane == 0) {
    for (uint32_t k = q_cnt > (uint32_t)C::QBUF ? q_cnt - C::QBUF : 0; k < q_cnt; ++k)
      mbar_drain(bar0 + 8 * (C::B_QFULL + k % C::QBUF), (k / C::QBUF) & 1);
  }
}

// KV producer warp: K and V tiles in the MMA's consumption order into the slot
// ring.  One TMA box is one page (or the part of a page inside the tile) of
// one KV head; lane k issues box k.  With bf16 pools both producers walk the
// order; this one issues the loads whose index has parity `which` and skips
// the others.  With E4M3 pools (F8) one producer (which = 2) issues every
// load, into the fp8 staging ring the converter warp drains.  Each lane reads
// its page id from the table right before its box (a loop-carried look-ahead
// of the ids made every producer wait on every load's table read).
template <int D, bool F8>
__device__ __forceinline__ void producer_role(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                              const AttnParams& p, uint32_t sKV, uint32_t bar0,
                                              int n_items, uint32_t which, volatile int* abort) {
  using C = TileCfg<D, F8>;
  constexpr int RING = F8 ? C::NST : C::NSLOT;
  constexpr int B_FULL = F8 ? C::B_STFULL : C::B_KVFULL;
  constexpr int B_EMPTY = F8 ? C::B_STEMPTY : C::B_KVEMPTY;
  constexpr int RING_BYTES = F8 ? C::STAGE_BYTES : C::SLOT_BYTES;
  constexpr int NCH = F8 ? D / 128 : C::DCH;   // boxes (128-byte column chunks) per page part
  constexpr int CH_ELEMS = F8 ? 128 : 64;      // elements of one chunk
  const int lane = threadIdx.x & 31;
  uint32_t ld_idx = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const int n = item_tiles(w, C::BN);
    for (int s = 0; s < 2 * n; ++s, ++ld_idx) {
      if (which < 2 && (ld_idx & 1u) != which) continue;
      int j;
      bool is_v;
      kv_sequence(s, n, j, is_v);
      const uint32_t slot = ld_idx % RING;
      if (!warp_wait(bar0 + 8 * (B_EMPTY + slot), ((ld_idx / RING) & 1) ^ 1, abort)) {
        ok = false;
        break;
      }
      const int n0 = w.kv_lo + j * C::BN;
      // every live row of the tile is loaded (rows past the item's causal limit
      // included) so that no stale shared memory meets P * V
      const int live = min(w.kv_len - n0, C::BN);
      const int nbox = (live + p.box_h - 1) >> p.box_log2;
      const uint32_t full = bar0 + 8 * (B_FULL + slot);
      if (lane == 0) mbar_arrive_expect_tx(full, nbox * p.box_h * 128 * NCH);
      __syncwarp();
      if (lane < nbox) {
        const int r = n0 + lane * p.box_h;     // < kv_len <= C * ps
        int page = __ldg(p.page_table + (size_t)w.b * p.tstride + (r >> p.ps_log2));
        if (page < 0 || (p.num_pages > 0 && page >= p.num_pages)) {
          atomicOr(p.status, kStatusBadPage);
          page = -1;   // out of the tensor map: the box reads as zeros
        }
        const CUtensorMap* tm = is_v ? tm_v : tm_k;
        const uint32_t dst = sKV + slot * RING_BYTES + lane * p.box_h * 128;
        for (int c = 0; c < NCH; ++c)
          tma_load_4d(dst + c * C::SLOT_CHUNK, tm, full, c * CH_ELEMS, w.kvh, r & (p.ps - 1),
                      page);
      }
    }
  }
  if (!ok || *abort) {
    // wait (bounded) for our copies still in flight before the CTA exits
    if (lane == 0) {
      const uint32_t first = ld_idx > (uint32_t)RING ? ld_idx - RING : 0;
      for (uint32_t k = first; k < ld_idx; ++k)
        if (which > 1 || (k & 1u) == which)
          mbar_drain(bar0 + 8 * (B_FULL + k % RING), (k / RING) & 1);
    }
  }
}

// E4M3 converter warp (F8).  Walks the producer's load order; staging tile
// i % NST holds load i as D / 128 chunks of 64 rows x 128 bytes (16-byte unit
// x of row r at x ^ (r & 7), the TMA 128-byte swizzle).  Each code is widened
// to fp16 with cvt.rn.f16x2.e4m3x2 (exact: every E4M3 value is an fp16 value)
// into 16-bit slot i % NSLOT, laid out as a TMA-loaded bf16 tile would be
// (64-column chunks, 128-byte swizzle), so the MMAs read it unchanged.  The 8
// lanes of a store phase take one 16-byte unit of 8 consecutive rows, whose
// swizzled places in the staging tile and in the slot fall in 8 distinct bank
// groups.  V rows at and past the request's end are written as zeros (P is 0
// there, but 0 * NaN is not); K rows there only meet masked scores.
template <int D>
__device__ __forceinline__ void convert_role(const AttnParams& p, uint32_t sKV, uint32_t sST,
                                             uint32_t bar0, int n_items, int cw,
                                             volatile int* abort) {
  using C = TileCfg<D, true>;
  constexpr int UPR = D / 16;                        // 16-byte fp8 units per row
  constexpr int UNITS = C::BN * UPR;
  const int lane = threadIdx.x & 31;
  uint32_t ld_idx = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const int n = item_tiles(w, C::BN);
    for (int s = 0; s < 2 * n; ++s, ++ld_idx) {
      int j;
      bool is_v;
      kv_sequence(s, n, j, is_v);
      const uint32_t st = ld_idx % C::NST, slot = ld_idx % C::NSLOT;
      if (!warp_wait(bar0 + 8 * (C::B_STFULL + st), (ld_idx / C::NST) & 1, abort) ||
          !warp_wait(bar0 + 8 * (C::B_KVEMPTY + slot), ((ld_idx / C::NSLOT) & 1) ^ 1, abort)) {
        ok = false;
        break;
      }
      const int n0 = w.kv_lo + j * C::BN;
      const int zero_from = is_v ? max(0, min(C::BN, w.kv_len - n0)) : C::BN;
      const uint32_t src0 = sST + st * C::STAGE_BYTES;
      const uint32_t dst0 = sKV + slot * C::SLOT_BYTES;
      // passes of 8 x 32 units, dealt round-robin to the NCONV widening warps
#pragma unroll 1
      for (int u0 = cw * 8 * 32; u0 < UNITS; u0 += C::NCONV * 8 * 32) {
        uint32_t x[8][4];
#pragma unroll
        for (int e = 0; e < 8; ++e) {                 // all loads of the pass first
          const int u = u0 + e * 32 + lane;
          const int row = (u & 7) + 8 * (u / (8 * UPR)), k = (u >> 3) % UPR;
          if (row < zero_from) {
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(x[e][0]), "=r"(x[e][1]), "=r"(x[e][2]), "=r"(x[e][3])
                         : "r"(src0 + (k >> 3) * C::SLOT_CHUNK + row * 128 +
                               (((k & 7) ^ (row & 7)) << 4)));
          } else {
            x[e][0] = x[e][1] = x[e][2] = x[e][3] = 0u;   // E4M3 code 0 is +0
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int u = u0 + e * 32 + lane;
          const int row = (u & 7) + 8 * (u / (8 * UPR)), k = (u >> 3) % UPR;
          uint32_t h[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) e4m3x4_to_f16x4(x[e][q], h[2 * q], h[2 * q + 1]);
          // halves 0-7 go to 16-byte unit 2 (k & 3) of the 64-column chunk
          // k / 4, halves 8-15 to the next unit (unit y stored at y ^ (row & 7))
          const uint32_t rbase = dst0 + (k >> 2) * C::SLOT_CHUNK + row * 128;
          const uint32_t y0 = 2 * (k & 3);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                           rbase + ((y0 ^ (row & 7)) << 4)),
                       "r"(h[0]), "r"(h[1]), "r"(h[2]), "r"(h[3])
                       : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                           rbase + (((y0 + 1) ^ (row & 7)) << 4)),
                       "r"(h[4]), "r"(h[5]), "r"(h[6]), "r"(h[7])
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar0 + 8 * (C::B_KVFULL + slot));
        mbar_arrive(bar0 + 8 * (C::B_STEMPTY + st));
      }
    }
  }
}

// MMA issuer.  bf16 operands, or fp16 ones with E4M3 pools (F8: Q rounded to
// fp16 by the Q loader, K and V widened by the converter, P written as fp16).
template <int D, bool F8>
__device__ __forceinline__ void mma_role(const AttnParams& p, uint32_t sQ, uint32_t sKV,
                                         uint32_t bar0, uint32_t tmem, int n_items,
                                         volatile int* abort) {
  using C = TileCfg<D, F8>;
  constexpr uint32_t kIdescS = F8 ? idesc_f16_f32(kBM, C::BN, false, false)
                                  : idesc_bf16_f32(kBM, C::BN, false, false);
  constexpr uint32_t kIdescPV = F8 ? idesc_f16_f32(kBM, D, false, true)
                                   : idesc_bf16_f32(kBM, D, false, true);
  uint32_t ld_idx = 0, g_base = 0, q_cnt = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const int n = item_tiles(w, C::BN);
    if (n == 0) continue;
    const uint32_t qb = q_cnt % C::QBUF;
    const uint32_t sQb = sQ + qb * C::Q_BYTES;
    const bool comp = item_compensated(w, p.causal);
    if (!warp_wait(bar0 + 8 * (C::B_QFULL + qb), (q_cnt / C::QBUF) & 1, abort)) { ok = false; break; }
    tc_fence_after();
    for (int s = 0; s < 2 * n; ++s) {
      int j;
      bool is_v;
      kv_sequence(s, n, j, is_v);
      const uint32_t slot = ld_idx % C::NSLOT;
      if (!warp_wait(bar0 + 8 * (C::B_KVFULL + slot), (ld_idx / C::NSLOT) & 1, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t slot_addr = sKV + slot * C::SLOT_BYTES;
      const uint32_t g = g_base + j, sb = g & 1;
      if (!is_v) {
        // S[sb] = Q K^T: K-major A (Q) and B (K), 16 columns of D per MMA
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(sQb + (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32, 16, 1024);
          const uint64_t bd =
              smem_desc_sw128(slot_addr + (kk >> 2) * C::SLOT_CHUNK + (kk & 3) * 32, 16, 1024);
          mma_ss_w(tmem + sb * C::BN, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit_w(bar0 + 8 * (C::B_SFULL + sb));
        tc_commit_w(bar0 + 8 * (C::B_KVEMPTY + slot));
        if (j == n - 1) tc_commit_w(bar0 + 8 * (C::B_QEMPTY + qb));
      } else {
        if (!warp_wait(bar0 + 8 * (C::B_PFULL + sb), (g >> 1) & 1, abort)) { ok = false; break; }
        if (j == 0 && !warp_wait(bar0 + 8 * C::B_OEMPTY, (q_cnt & 1) ^ 1, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // O += P V: A = P (bf16, packed two per TMEM column), B = V tile (MN-major:
        // D contiguous), 16 keys per MMA
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t bd = smem_desc_sw128(slot_addr + kk * 16 * 128, C::SLOT_CHUNK, 1024);
          mma_ts_w(tmem + C::O_COL, tmem + sb * C::BN + kk * 8, bd, kIdescPV,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
        if (comp) {
          // O += P_lo V: the rounding remainder of P sits in the second half of
          // the S buffer (columns BN / 2 .. BN - 1)
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(slot_addr + kk * 16 * 128, C::SLOT_CHUNK, 1024);
            mma_ts_w(tmem + C::O_COL, tmem + sb * C::BN + C::BN / 2 + kk * 8, bd, kIdescPV, 1u);
          }
        }
        tc_commit_w(bar0 + 8 * (C::B_PVDONE + sb));
        tc_commit_w(bar0 + 8 * (C::B_KVEMPTY + slot));
      }
      ++ld_idx;
    }
    g_base += n;
    ++q_cnt;
  }
  // all MMAs issued by this warp complete before TMEM is released
  tc_commit_w(bar0 + 8 * C::B_DRAIN);
  if ((threadIdx.x & 31) == 0) mbar_drain(bar0 + 8 * C::B_DRAIN, 0);
  __syncwarp();
}

// P = exp2(s * scale_log2 - m) of one row of a BN-key tile, packed as bf16
// pairs (fp16 with F16) into TMEM columns [taddr, taddr + BN/2); with COMP the
// rounding remainder P_lo = 16-bit(P - P_hi) goes to [taddr + BN/2, taddr + BN).
// Returns the row sum of the fp32 P.  (The caller waits for the stores.)
template <int BN, bool COMP, bool F16 = false>
__device__ __forceinline__ float write_p(float (&s)[BN], float scale_log2, float m_use,
                                         uint32_t taddr) {
  // s * scale_log2 - m and the row sum in packed fp32 pairs (half the
  // instructions); the sum runs in two independent pair accumulators
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m_use, -m_use);
  uint64_t rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
  uint32_t pk[BN / 2];
#pragma unroll
  for (int c = 0; c < BN; c += 2) {
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sc2, nm2), x0, x1);
    const float p0 = ex2_approx(x0);
    const float p1 = ex2_approx(x1);
    rs2[(c >> 1) & 1] = f2_add(rs2[(c >> 1) & 1], f2_pack(p0, p1));
    pk[c >> 1] = F16 ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
    if constexpr (COMP) {
      s[c] = p0;
      s[c + 1] = p1;
    }
  }
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) tmem_st16(taddr + c * 16, pk + c * 16);
  if constexpr (COMP) {
#pragma unroll
    for (int c = 0; c < BN; c += 2) {
      if constexpr (F16)
        pk[c >> 1] = pack_f16x2(s[c] - f16_to_f32((unsigned short)(pk[c >> 1] & 0xffffu)),
                                s[c + 1] - f16_to_f32((unsigned short)(pk[c >> 1] >> 16)));
      else
        pk[c >> 1] = pack_bf16x2(s[c] - bf16_to_f32(pk[c >> 1] & 0xffffu),
                                 s[c + 1] - bf16_to_f32(pk[c >> 1] >> 16));
    }
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) tmem_st16(taddr + BN / 2 + c * 16, pk + c * 16);
  }
  float a0, a1, b0, b1;
  f2_unpack(rs2[0], a0, a1);
  f2_unpack(rs2[1], b0, b1);
  return (a0 + b0) + (a1 + b1);
}

template <int D, bool F8>
__device__ __forceinline__ void softmax_role(const CUtensorMap* tm_o, const AttnParams& p,
                                             uint32_t sKV, uint32_t sEpi, uint32_t bar0,
                                             uint32_t tmem, int n_items, volatile int* merge_flag,
                                             volatile int* abort) {
  using C = TileCfg<D, F8>;
  constexpr int BN = C::BN;
  const int r = threadIdx.x;          // query row of the tile, 0..127
  const int warp = r >> 5, lane = r & 31;
  const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);   // this warp's lanes
  const int G = p.G;
  const int T = p.cu_q_lens ? __ldg(p.cu_q_lens + p.B) : p.B;
  const uint32_t sEpiW = sEpi + warp * C::EPI_WARP_BYTES;
  uint32_t g_base = 0, ld_base = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const int n = item_tiles(w, BN);
    const int n_rows = w.n_tok * G;
    const bool real = r < n_rows;
    const bool warp_active = warp * 32 < n_rows;
    const int t = w.t_base + w.q_tok0 + r / G;
    const int h = w.kvh * G + r % G;
    const bool split = w.n_splits > 1;
    const bool comp = item_compensated(w, p.causal);
    const size_t prow = ((((size_t)w.b * p.Hkv + w.kvh) * p.S_max + w.split) * kBM + r);
    if (n == 0) {
      // no key is visible to any row of the block: O = 0, LSE = -inf
      if (real) {
        if (split) {
          float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D);
          for (int c = 0; c < D / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          p.part_lse[prow] = -INFINITY;
        } else {
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)t * p.Hq + h) * D);
          for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          if (p.lse) p.lse[(size_t)t * p.Hq + h] = -INFINITY;
        }
      }
      if (split && p.fused_merge)
        split_arrive_and_merge(p, w, D, bar0 + 8 * C::B_MERGE, merge_flag, abort);
      continue;
    }
    // keys visible to this row: [kv_lo, lim)
    const int i_r = w.q_tok0 + r / G;
    const int lim = p.causal ? min(w.kv_hi, i_r + (w.kv_len - w.q_len) + 1) : w.kv_hi;
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = 0; j < n && ok; ++j) {
      const uint32_t g = g_base + j, sb = g & 1;
      if (!warp_wait(bar0 + 8 * (C::B_SFULL + sb), (g >> 1) & 1, abort)) { ok = false; break; }
      tc_fence_after();
      const int n0 = w.kv_lo + j * BN;
      if (warp_active) {
        float s[BN];
        {
          uint32_t v[BN / 32][32];
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) tmem_ld32(trow + sb * BN + c * 32, v[c]);
          tmem_ld_wait(v[0]);
#pragma unroll
          for (int c = 1; c < BN / 32; ++c) reg_tie(v[c]);
#pragma unroll
          for (int c = 0; c < BN / 32; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(v[c][e]);
        }
        const int nvis = lim - n0;
        if (nvis < BN) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= nvis) s[c] = -INFINITY;   // mask by select, never by add
        }
        // row maximum: four independent chains of three-input maxima
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < BN; c += 8) {
#pragma unroll
          for (int k = 0; k < 4; ++k) mx4[k] = fmax3(mx4[k], s[c + 2 * k], s[c + 2 * k + 1]);
        }
        const float mx = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        const bool need = real && (m_new > m_run + kRescaleThreshold);
        if (j > 0 && __any_sync(0xffffffffu, need && m_run != -INFINITY)) {
          // O holds the sum up to tile g-1: wait for that P V, then rescale it
          const uint32_t gp = g - 1;
          if (!warp_wait(bar0 + 8 * (C::B_PVDONE + (gp & 1)), (gp >> 1) & 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = need ? ex2_approx(m_run - m_new) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < D / 32; c += C::OCH) {
            uint32_t v[C::OCH][32];
#pragma unroll
            for (int h2 = 0; h2 < C::OCH; ++h2) tmem_ld32(trow + C::O_COL + (c + h2) * 32, v[h2]);
            tmem_ld_wait(v[0]);
#pragma unroll
            for (int h2 = 1; h2 < C::OCH; ++h2) reg_tie(v[h2]);
#pragma unroll
            for (int h2 = 0; h2 < C::OCH; ++h2) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                v[h2][e] = __float_as_uint(__uint_as_float(v[h2][e]) * alpha);
              tmem_st32(trow + C::O_COL + (c + h2) * 32, v[h2]);
            }
          }
          tmem_st_wait();
        }
        if (need) {
          l_run *= ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        // P overwrites the first BN/2 columns of the S buffer it came from
        // (compensated items: P_lo the other BN/2); item-uniform branch, each
        // side its own instance so the common one stays as lean as before
        l_run += comp ? write_p<BN, true, F8>(s, p.scale_log2, m_use, trow + sb * BN)
                      : write_p<BN, false, F8>(s, p.scale_log2, m_use, trow + sb * BN);
        tmem_st_wait();
      }
      if (j == n - 1) {
        if (!F8 && n0 + BN > w.kv_len) {
          // Last tile of the request: rows at and past kv_len in the V tile are
          // tail slots or rows never loaded; zero them so that 0 * garbage
          // cannot reach O (P is 0 there, but 0 * NaN is NaN).  (The E4M3
          // converter writes those rows as zeros itself.)
          const uint32_t ldv = ld_base + 2 * n - 1;
          const uint32_t slot = ldv % C::NSLOT;
          if (!warp_wait(bar0 + 8 * (C::B_KVFULL + slot), (ldv / C::NSLOT) & 1, abort)) {
            ok = false;
            break;
          }
          const int z0 = w.kv_len - n0;
          const int units = (BN - z0) * C::DCH * 8;
          const uint32_t base = sKV + slot * C::SLOT_BYTES;
          for (int u = r; u < units; u += 128) {
            const int row = z0 + u / (C::DCH * 8);
            const int rem = u % (C::DCH * 8);
            const uint32_t a = base + (rem >> 3) * C::SLOT_CHUNK + row * 128 + (rem & 7) * 16;
            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0) : "memory");
          }
          fence_proxy_async_smem();
        }
        // make sure the P V of the previous tile has completed before this
        // tile's P is published (keeps pv_done phases unambiguous)
        const uint32_t gp = g - 1;
        if (!warp_wait(bar0 + 8 * (C::B_PVDONE + (gp & 1)), (gp >> 1) & 1, abort)) {
          ok = false;
          break;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar0 + 8 * (C::B_PFULL + sb));
    }
    if (!ok) break;
    // ---- epilogue: O / l -> out (or the split partial), LSE
    const uint32_t gl = g_base + n - 1;
    if (!warp_wait(bar0 + 8 * (C::B_PVDONE + (gl & 1)), (gl >> 1) & 1, abort)) { ok = false; break; }
    tc_fence_after();
    if (warp_active) {
      const float inv_l = l_run > 0.f ? p.v_scale / l_run : 0.f;   // V descale (1 for bf16)
      const float lse_v = l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      // whole blocks of 32 / G tokens per warp go out through TMA stores
      const bool o_tma = C::EPI_BYTES > 0 && !split && p.o_tma && w.n_tok == p.tpb &&
                         w.t_base + w.q_tok0 + p.tpb <= T;
      const int t_w0 = w.t_base + w.q_tok0 + warp * (32 / G);
#pragma unroll 1
      for (int c = 0; c < D / 32; c += C::OCH) {
        uint32_t vv[C::OCH][32];
#pragma unroll
        for (int h2 = 0; h2 < C::OCH; ++h2) tmem_ld32(trow + C::O_COL + (c + h2) * 32, vv[h2]);
        tmem_ld_wait(vv[0]);
#pragma unroll
        for (int h2 = 1; h2 < C::OCH; ++h2) reg_tie(vv[h2]);
        if (real) {
#pragma unroll
          for (int h2 = 0; h2 < C::OCH; ++h2) {
            const uint32_t* v = vv[h2];
            if (split) {
              float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D + (c + h2) * 32);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(v[4 * e]) * inv_l,
                                     __uint_as_float(v[4 * e + 1]) * inv_l,
                                     __uint_as_float(v[4 * e + 2]) * inv_l,
                                     __uint_as_float(v[4 * e + 3]) * inv_l);
            } else if (o_tma) {
              // 32 rows x 32 columns staged in the 64-byte swizzle of the out
              // tensor map, then written by one TMA store per warp (full
              // 64-byte row pieces instead of one 16-byte piece per row)
              if (lane == 0) bulk_wait_read_all();   // previous store has read the buffer
              __syncwarp();
              const uint32_t row_addr = sEpiW + lane * 64;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const uint32_t a = row_addr + ((e ^ ((lane >> 1) & 3)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                             "r"(pack_bf16x2(__uint_as_float(v[8 * e + 0]) * inv_l, __uint_as_float(v[8 * e + 1]) * inv_l)),
                             "r"(pack_bf16x2(__uint_as_float(v[8 * e + 2]) * inv_l, __uint_as_float(v[8 * e + 3]) * inv_l)),
                             "r"(pack_bf16x2(__uint_as_float(v[8 * e + 4]) * inv_l, __uint_as_float(v[8 * e + 5]) * inv_l)),
                             "r"(pack_bf16x2(__uint_as_float(v[8 * e + 6]) * inv_l, __uint_as_float(v[8 * e + 7]) * inv_l))
                             : "memory");
              }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_3d(tm_o, sEpiW, (c + h2) * 32, w.kvh * G, t_w0);
                bulk_commit_group();
              }
            } else {
              uint4* dst =
                  reinterpret_cast<uint4*>(p.out + ((size_t)t * p.Hq + h) * D + (c + h2) * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint4 q4;
                q4.x = pack_bf16x2(__uint_as_float(v[8 * e + 0]) * inv_l, __uint_as_float(v[8 * e + 1]) * inv_l);
                q4.y = pack_bf16x2(__uint_as_float(v[8 * e + 2]) * inv_l, __uint_as_float(v[8 * e + 3]) * inv_l);
                q4.z = pack_bf16x2(__uint_as_float(v[8 * e + 4]) * inv_l, __uint_as_float(v[8 * e + 5]) * inv_l);
                q4.w = pack_bf16x2(__uint_as_float(v[8 * e + 6]) * inv_l, __uint_as_float(v[8 * e + 7]) * inv_l);
                dst[e] = q4;
              }
            }
          }
        }
      }
      if (real) {
        if (split) p.part_lse[prow] = lse_v;
        else if (p.lse) p.lse[(size_t)t * p.Hq + h] = lse_v;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar0 + 8 * C::B_OEMPTY);
    if (split && p.fused_merge)
        split_arrive_and_merge(p, w, D, bar0 + 8 * C::B_MERGE, merge_flag, abort);
    g_base += n;
    ld_base += 2 * n;
  }
  if (lane == 0) bulk_wait_all();   // O stores complete before the CTA exits
}

template <int D, bool F8 = false>
__global__ void __maxnreg__((TileCfg<D, F8>::MAXREG))
    pa_attention_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_o, const AttnParams p) {
  using C = TileCfg<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;             // 1024-B aligned for SW128
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sQ = base;
  const uint32_t sKV = base + C::QBUF * C::Q_BYTES;
  const uint32_t sST = sKV + C::NSLOT * C::SLOT_BYTES;     // fp8 staging (F8 only)
  const uint32_t sEpi = sST + C::NST * C::STAGE_BYTES;
  const uint32_t bar0 = sEpi + C::EPI_BYTES;
  uint8_t* bar_ptr = smem + (bar0 - base);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ptr + 8 * C::NBAR);
  volatile int* abort = reinterpret_cast<volatile int*>(bar_ptr + 8 * C::NBAR + 4);
  volatile int* merge_flag = reinterpret_cast<volatile int*>(bar_ptr + 8 * C::NBAR + 8);

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(bar0 + 8 * C::B_MERGE, kSoftmaxWarps);
    for (int i = 0; i < C::QBUF; ++i) {
      mbar_init(bar0 + 8 * (C::B_QFULL + i), 1);
      mbar_init(bar0 + 8 * (C::B_QEMPTY + i), 1);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      // filled by TMA (one expect_tx arrival) or by the NCONV widening warps (F8)
      mbar_init(bar0 + 8 * (C::B_KVFULL + i), F8 ? C::NCONV : 1);
      mbar_init(bar0 + 8 * (C::B_KVEMPTY + i), 1);
    }
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(bar0 + 8 * (C::B_STFULL + i), 1);
      mbar_init(bar0 + 8 * (C::B_STEMPTY + i), C::NCONV);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar0 + 8 * (C::B_SFULL + i), 1);
      mbar_init(bar0 + 8 * (C::B_PFULL + i), 4);
      mbar_init(bar0 + 8 * (C::B_PVDONE + i), 1);
    }
    mbar_init(bar0 + 8 * C::B_OEMPTY, 4);
    mbar_init(bar0 + 8 * C::B_DRAIN, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  constexpr bool two_producers = !F8 || C::NCONV > 1;
  if ((warp == kProducerWarp || (two_producers && warp == kProducer2Warp)) &&
      (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (!F8 && warp == kQWarp && (threadIdx.x & 31) == 0) tma_prefetch_desc(&tm_q);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything above overlaps the scheduler kernel; its work list is read below
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int n_items = list_count(p);

  bool widening_warp = false;
  if constexpr (F8 && C::NCONV > 1) {
    // E4M3, D = 256: warps 8-11 widen each staged tile together
    if (warp >= 8) {
      convert_role<D>(p, sKV, sST, bar0, n_items, warp - 8, abort);
      widening_warp = true;
    }
  }
  if (widening_warp) {
  } else if (warp == kProducerWarp || warp == kProducer2Warp) {
    if constexpr (F8 && C::NCONV > 1) {
      // two producers, one parity of the loads (and one staging tile) each
      producer_role<D, true>(&tm_k, &tm_v, p, sST, bar0, n_items,
                             warp == kProducerWarp ? 0u : 1u, abort);
    } else if constexpr (F8) {
      // one producer issues every load into the staging ring; the other warp
      // widens the staged tiles into the 16-bit slots
      if (warp == kProducerWarp) producer_role<D, true>(&tm_k, &tm_v, p, sST, bar0, n_items, 2u, abort);
      else convert_role<D>(p, sKV, sST, bar0, n_items, 0, abort);
    } else {
      producer_role<D, false>(&tm_k, &tm_v, p, sKV, bar0, n_items,
                              warp == kProducerWarp ? 0u : 1u, abort);
    }
  } else if (warp == kQWarp) {
    q_loader_role<D, F8>(&tm_q, p, sQ, bar0, n_items, abort);
  } else if (warp == kMmaWarp) {
    mma_role<D, F8>(p, sQ, sKV, bar0, tmem, n_items, abort);   // all 32 lanes
  } else {
    softmax_role<D, F8>(&tm_o, p, sKV, sEpi, bar0, tmem, n_items, merge_flag, abort);
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(p.status, kStatusTimeout);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// =========================================================================== merge
struct MergeParams {
  const int4* req_info;  // {n_splits, q_len, t_base, kv_len}
  const int* split_list;
  const WsHeader* hdr;
  const float* part_o;
  const float* part_lse;
  uint16_t* out;
  float* lse;
  int B, Hq, Hkv, G, D, S_max;
};

// out = sum_s exp(lse_s - L) O_s with L = ln sum_s exp(lse_s): the exact merge
// of attention states over disjoint key ranges; empty splits (lse_s = -inf)
// get weight 0.  One warp per (split request, KV head, row); the loads of
// several splits are kept in flight together.
__global__ void __launch_bounds__(128) pa_merge_kernel(MergeParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int n_req = p.hdr->n_split_reqs;
  const int warp = threadIdx.x >> 5;
  // row-major over (request, KV head): unit u is row u / n_kh of block u % n_kh,
  // so the live rows (r < q_len * G) come first and spread over all warps
  const int n_kh = n_req * p.Hkv;
  const int n_units = n_kh * kBM;
  for (int u = blockIdx.x * 4 + warp; u < n_units; u += gridDim.x * 4) {
    const int r = u / n_kh;
    const int kh = u % n_kh;
    const int kvh = kh % p.Hkv;
    const int b = p.split_list[kh / p.Hkv];
    const int4 ri = p.req_info[b];
    const int ns = ri.x;
    if (r >= ri.y * p.G) continue;
    const size_t base = ((size_t)b * p.Hkv + kvh) * p.S_max * kBM + r;   // + s * kBM
    const int t = ri.z + r / p.G;
    const int h = kvh * p.G + r % p.G;
    merge_one_row(p.part_o, p.part_lse, base, ns, p.D, p.out + ((size_t)t * p.Hq + h) * p.D,
                  p.lse ? p.lse + (size_t)t * p.Hq + h : nullptr);
  }
}

// Self-test of the bounded waits (pa_selftest_wait_timeout).  One CTA of
// three warps and two mbarriers that nothing ever arrives at.  Warp 1 waits on
// the first with a short limit, gives up, sets the CTA's abort flag and the
// timeout status bit; warp 2 waits on the second with the production limit
// and must leave through the abort shortcut long before that limit.  Both
// record how long they waited (microseconds of global time).
__global__ void __launch_bounds__(96) pa_selftest_wait_kernel(unsigned* status, uint64_t limit_ns,
                                                               unsigned* elapsed_us) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &abort_flag;
  if (warp == 1 || warp == 2) {
    const uint64_t t0 = global_timer_ns();
    const bool ok = __all_sync(0xffffffffu,
                               mbar_wait_for(smem_u32(&bars[warp - 1]), 0, abort,
                                             warp == 1 ? limit_ns : kWaitTimeoutNs));
    const uint64_t dt = global_timer_ns() - t0;
    if (lane == 0) {
      elapsed_us[warp - 1] = (unsigned)(dt / 1000u);
      if (!ok) atomicOr(status, kStatusTimeout);
    }
  }
  __syncthreads();
}

}  // namespace pa
