// pa_prefill.cuh -- two-stage prefill attention kernel (sm_100a, head_dim 64/128).
//
// A work item here is a PAIR of consecutive 128-row query blocks of one
// (request, KV head): stage A holds query tokens [q0, q0 + tpb), stage B the
// next tpb tokens (possibly partial or empty).  Both stages read the same K/V
// tiles, so every tile loaded feeds 256 query rows: half the K/V traffic per
// row of the one-stage kernel.  The MMA warp alternates between the stages
// ("ping-pong"): while the softmax warpgroup of one stage works on its scores,
// the tensor core computes P V and the next S = Q K^T of the other stage.  This
// follows the two-query-stage (q_stage = 2) SM100 prefill configuration that
// "[Perf][FA4] Warm up dense (paged) FA4 attention kernels" (vLLM PR #48156,
// review thread) describes, written here from that description.
//
// Q lives in tensor memory.  Q is read once per item, so it always comes from
// DRAM; with one CTA per SM a Q tile held in shared memory for the whole item
// would leave either no room to load the next item's Q early or too little
// room for the K/V ring.  Here the Q loader fills a shared-memory staging
// buffer, the softmax warps copy their stage's rows into TMEM at the start of
// the item and release the staging buffer at once, so the next item's Q loads
// while the current item runs.  S = Q K^T then takes A from TMEM.
//
// Roles (11 warps, one CTA per SM):
//   warps 0-3   stage A: Q copy to TMEM, softmax, correction, epilogue
//   warps 4-7   the same for stage B
//   warp  8     K/V producer (page-table-driven TMA, order K0 V0 K1 V1 ...)
//   warp  9     MMA issuer (one thread)
//   warp  10    Q loader
// TMEM (512 columns): S_A, S_B (BN each), O_A, O_B (D each), Q_A, Q_B (D/2 each).
// Each stage has a single S buffer: S_X(j+1) is issued after P_X(j) V(j), so
// the completion of S_X(j+1) also guarantees that P_X(j) V(j) has completed.
#pragma once

#include "pa_kernels.cuh"

namespace pa {

template <int D>
struct PairCfg {
  static_assert(D == 64 || D == 128, "two-stage kernel: head_dim 64 or 128");
  static constexpr int BN = 64;
  static constexpr int DCH = D / 64;
  static constexpr int Q_CHUNK = kBM * 128;
  static constexpr int Q_BYTES = kBM * D * 2;          // one stage
  static constexpr int SLOT_CHUNK = BN * 128;
  static constexpr int SLOT_BYTES = BN * D * 2;
  static constexpr int NSLOT = (D == 64) ? 16 : 10;
  static constexpr int S_COL = 0;                      // + stage * BN
  static constexpr int O_COL = 2 * BN;                 // + stage * D
  static constexpr int Q_COL = 2 * BN + 2 * D;         // + stage * D / 2
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 352;
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, Q_WARP = 10;
  // barriers: q_full, q_smem_empty, q_tmem[2], kv_full[NSLOT], kv_empty[NSLOT],
  //           s_full[2], p_full[2], pv_done[2], o_empty[2], drain
  static constexpr int B_QFULL = 0, B_QSMEM = 1, B_QTMEM = 2, B_KVFULL = 4,
                       B_KVEMPTY = 4 + NSLOT, B_SFULL = 4 + 2 * NSLOT, B_PFULL = B_SFULL + 2,
                       B_PVDONE = B_PFULL + 2, B_OEMPTY = B_PVDONE + 2, B_DRAIN = B_OEMPTY + 2,
                       NBAR = B_DRAIN + 1;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_BYTES = 1024 + 2 * Q_BYTES + NSLOT * SLOT_BYTES + BAR_BYTES;
  static_assert(NBAR * 8 + 16 <= BAR_BYTES, "barrier area");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(Q_COL + D <= TMEM_COLS, "TMEM columns");
};

// Tokens of the two stages and KV tiles each needs.
struct PairShape {
  int tok[2];     // query tokens of stage A and B
  int lim[2];     // keys visible to the stage's last row (causal, end aligned)
  int nt[2];      // KV tiles of each stage (0 = the stage has nothing to do)
  int n;          // KV tiles of the item (max of the two)
};

__device__ __forceinline__ PairShape pair_shape(const WorkItem& w, int tpb, int BN) {
  PairShape s;
  s.tok[0] = max(0, min(tpb, w.q_len - w.q_tok0));
  s.tok[1] = max(0, min(tpb, w.q_len - w.q_tok0 - s.tok[0]));
  for (int x = 0; x < 2; ++x) {
    const int q0 = w.q_tok0 + x * tpb;
    int hi = q0 + s.tok[x] + (w.kv_len - w.q_len);
    hi = hi < 0 ? 0 : (hi > w.kv_len ? w.kv_len : hi);
    s.lim[x] = hi;
    s.nt[x] = s.tok[x] > 0 ? ceil_div(hi, BN) : 0;
  }
  s.n = max(s.nt[0], s.nt[1]);
  return s;
}

template <int D>
__device__ __forceinline__ void pair_q_loader(const CUtensorMap* tm_q, const AttnParams& p,
                                              uint32_t sQ, uint32_t bar0, int n_items,
                                              volatile int* abort) {
  using C = PairCfg<D>;
  const int lane = threadIdx.x & 31;
  const int G = p.G;
  const int T = p.cu_q_lens ? p.cu_q_lens[p.B] : p.B;
  uint32_t q_cnt = 0;
  ItemStream items(p.items, n_items, p.tpb);
  WorkItem w;
  while (items.next(w)) {
    const PairShape ps = pair_shape(w, p.tpb, C::BN);
    if (ps.n == 0) continue;
    // the staging buffer is free once all eight softmax warps copied the last Q
    if (!warp_wait(bar0 + 8 * C::B_QSMEM, (q_cnt & 1) ^ 1, abort)) break;
    const uint32_t qfull = bar0 + 8 * C::B_QFULL;
    const uint32_t sQb = sQ;
    bool tma[2];
    uint32_t tma_bytes = 0;
    for (int x = 0; x < 2; ++x) {
      const int t0 = w.t_base + w.q_tok0 + x * p.tpb;
      tma[x] = ps.tok[x] == p.tpb && t0 + p.tpb <= T;
      if (tma[x]) tma_bytes += C::DCH * p.tpb * G * 128;
    }
    if (lane == 0) {
      if (tma_bytes) mbar_expect_tx(qfull, tma_bytes);
      for (int x = 0; x < 2; ++x)
        if (tma[x])
          for (int c = 0; c < C::DCH; ++c)
            tma_load_3d(sQb + x * C::Q_BYTES + c * C::Q_CHUNK, tm_q, qfull, c * 64, w.kvh * G,
                        w.t_base + w.q_tok0 + x * p.tpb);
    }
    // partial blocks: plain loads of the live rows, stored with the TMA's swizzle
    for (int x = 0; x < 2; ++x) {
      if (tma[x] || ps.tok[x] == 0) continue;
      const int t0 = w.t_base + w.q_tok0 + x * p.tpb;
      const uint32_t base = sQb + x * C::Q_BYTES;
      const int units = ps.tok[x] * G * (D / 8);
      for (int u0 = 0; u0 < units; u0 += 8 * 32) {
        uint4 v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
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
                base + (c16 >> 3) * C::Q_CHUNK + r * 128 + (((c16 & 7) ^ (r & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[k].x),
                         "r"(v[k].y), "r"(v[k].z), "r"(v[k].w)
                         : "memory");
          }
        }
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(qfull);
    ++q_cnt;
    // Q is read once, so it always comes from DRAM; pull the next item's Q
    // into L2 now so that its load at the next item boundary is short.
    WorkItem nw;
    if (lane == 0 && items.peek(nw)) {
      for (int x = 0; x < 2; ++x) {
        const int t0 = nw.t_base + nw.q_tok0 + x * p.tpb;
        if (nw.q_len - nw.q_tok0 - x * p.tpb >= p.tpb && t0 + p.tpb <= T)
          for (int c = 0; c < C::DCH; ++c) tma_prefetch_l2_3d(tm_q, c * 64, nw.kvh * G, t0);
      }
    }
  }
  if (*abort && lane == 0 && q_cnt > 0) mbar_drain(bar0 + 8 * C::B_QFULL, (q_cnt - 1) & 1);
}

// K/V producer: tile j of an item is loaded as K_j then V_j (load index 2j and
// 2j + 1 of the item); every live row of the tile is loaded.  Page ids are
// loop-carried: the ids of tile j + 1 are fetched after K_j is issued and used
// one step later.
template <int D>
__device__ __forceinline__ void pair_producer(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                              const AttnParams& p, uint32_t sKV, uint32_t bar0,
                                              int n_items, volatile int* abort) {
  using C = PairCfg<D>;
  const int lane = threadIdx.x & 31;
  uint32_t ld_idx = 0;
  bool ok = true;
  int pid_next = 0;
  bool have_next = false;
  ItemStream items(p.items, n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const PairShape ps = pair_shape(w, p.tpb, C::BN);
    const int n = ps.n;
    if (n == 0) {
      have_next = false;
      continue;
    }
    int pid_k = have_next ? pid_next : tile_page_id(p, w, 0, C::BN, lane);
    int pid_v = 0;
    have_next = false;
    for (int s = 0; s < 2 * n; ++s) {
      const int j = s >> 1;
      const bool is_v = s & 1;
      const uint32_t slot = ld_idx % C::NSLOT;
      if (!warp_wait(bar0 + 8 * (C::B_KVEMPTY + slot), ((ld_idx / C::NSLOT) & 1) ^ 1, abort)) {
        ok = false;
        break;
      }
      const int n0 = j * C::BN;
      const int live = min(w.kv_len - n0, C::BN);
      const int nbox = ceil_div(live, p.box_h);
      const uint32_t full = bar0 + 8 * (C::B_KVFULL + slot);
      if (lane == 0) mbar_arrive_expect_tx(full, nbox * p.box_h * 128 * C::DCH);
      __syncwarp();
      int page;
      if (!is_v) {
        page = pid_k;
        pid_v = pid_k;
      } else {
        page = pid_v;
      }
      if (lane < nbox) {
        const int row = (n0 + lane * p.box_h) % p.ps;
        if (page < 0 || (p.num_pages > 0 && page >= p.num_pages)) {
          atomicOr(p.status, kStatusBadPage);
          page = -1;   // out of the tensor map: the box reads as zeros
        }
        const CUtensorMap* tm = is_v ? tm_v : tm_k;
        const uint32_t dst = sKV + slot * C::SLOT_BYTES + lane * p.box_h * 128;
        for (int c = 0; c < C::DCH; ++c)
          tma_load_4d(dst + c * C::SLOT_CHUNK, tm, full, c * 64, w.kvh, row, page);
      }
      if (!is_v) {
        if (j + 1 < n) {
          pid_k = tile_page_id(p, w, j + 1, C::BN, lane);
        } else {
          WorkItem nw;
          if (items.peek(nw) && pair_shape(nw, p.tpb, C::BN).n > 0) {
            pid_next = tile_page_id(p, nw, 0, C::BN, lane);
            have_next = true;
          }
        }
      }
      ++ld_idx;
    }
  }
  if (!ok || *abort) {
    if (lane == 0) {
      const uint32_t first = ld_idx > (uint32_t)C::NSLOT ? ld_idx - C::NSLOT : 0;
      for (uint32_t k = first; k < ld_idx; ++k)
        mbar_drain(bar0 + 8 * (C::B_KVFULL + k % C::NSLOT), (k / C::NSLOT) & 1);
    }
  }
}

// MMA issuer.  Per item (n tiles, stage X uses tiles j < nt[X]):
//   S_A(0), S_B(0)
//   for j: P_A(j) V(j); S_A(j+1); P_B(j) V(j); S_B(j+1)
// so the tensor core works on one stage while the other stage's softmax runs.
// S_X = Q_X K^T with Q_X read from TMEM; P_X V with P_X read from TMEM.
template <int D>
__device__ __forceinline__ void pair_mma(const AttnParams& p, uint32_t sKV, uint32_t bar0,
                                         uint32_t tmem, int n_items, volatile int* abort) {
  using C = PairCfg<D>;
  constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, C::BN, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, false, true);
  uint32_t ld_base = 0;
  uint32_t g[2] = {0, 0};     // tiles processed per stage (phase counters)
  uint32_t itc[2] = {0, 0};   // items per stage that had tiles (q_tmem / o_empty phases)
  bool ok = true;
  ItemStream items(p.items, n_items, p.tpb);
  WorkItem w;

  auto kv_wait = [&](uint32_t idx) -> bool {
    const uint32_t slot = idx % C::NSLOT;
    if (!mbar_wait(bar0 + 8 * (C::B_KVFULL + slot), (idx / C::NSLOT) & 1, abort)) return false;
    tc_fence_after();
    return true;
  };
  auto issue_s = [&](int x, uint32_t k_idx) {
    const uint32_t slot_addr = sKV + (k_idx % C::NSLOT) * C::SLOT_BYTES;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t bd =
          smem_desc_sw128(slot_addr + (kk >> 2) * C::SLOT_CHUNK + (kk & 3) * 32, 16, 1024);
      mma_ts(tmem + C::S_COL + x * C::BN, tmem + C::Q_COL + x * (D / 2) + kk * 8, bd, kIdescS,
             kk > 0 ? 1u : 0u);
    }
    tc_commit(bar0 + 8 * (C::B_SFULL + x));
  };
  auto issue_pv = [&](int x, uint32_t v_idx, bool first) {
    const uint32_t slot_addr = sKV + (v_idx % C::NSLOT) * C::SLOT_BYTES;
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk) {
      const uint64_t bd = smem_desc_sw128(slot_addr + kk * 16 * 128, C::SLOT_CHUNK, 1024);
      mma_ts(tmem + C::O_COL + x * D, tmem + C::S_COL + x * C::BN + kk * 8, bd, kIdescPV,
             (!first || kk > 0) ? 1u : 0u);
    }
    tc_commit(bar0 + 8 * (C::B_PVDONE + x));
  };

  while (ok && items.next(w)) {
    const PairShape ps = pair_shape(w, p.tpb, C::BN);
    const int n = ps.n;
    if (n == 0) continue;
    // Q of each working stage copied into TMEM by its softmax warps
    for (int x = 0; x < 2 && ok; ++x)
      if (ps.nt[x] > 0 && !mbar_wait(bar0 + 8 * (C::B_QTMEM + x), itc[x] & 1, abort)) ok = false;
    if (!ok) break;
    tc_fence_after();
    // tile 0: S of both stages
    if (!kv_wait(ld_base)) { ok = false; break; }
    for (int x = 0; x < 2; ++x)
      if (ps.nt[x] > 0) issue_s(x, ld_base);
    tc_commit(bar0 + 8 * (C::B_KVEMPTY + ld_base % C::NSLOT));
    for (int j = 0; j < n && ok; ++j) {
      const uint32_t v_idx = ld_base + 2 * j + 1, k_next = ld_base + 2 * j + 2;
      if (!kv_wait(v_idx)) { ok = false; break; }
      bool k_ready = false;
      for (int x = 0; x < 2; ++x) {
        if (j < ps.nt[x]) {
          if (!mbar_wait(bar0 + 8 * (C::B_PFULL + x), (g[x] + j) & 1, abort)) { ok = false; break; }
          if (j == 0 && !mbar_wait(bar0 + 8 * (C::B_OEMPTY + x), (itc[x] & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(x, v_idx, j == 0);
        }
        if (x == 1) tc_commit(bar0 + 8 * (C::B_KVEMPTY + v_idx % C::NSLOT));
        if (j + 1 < n) {
          if (!k_ready) {
            if (!kv_wait(k_next)) { ok = false; break; }
            k_ready = true;
          }
          if (j + 1 < ps.nt[x]) issue_s(x, k_next);
          if (x == 1) tc_commit(bar0 + 8 * (C::B_KVEMPTY + k_next % C::NSLOT));
        }
      }
    }
    for (int x = 0; x < 2; ++x) {
      g[x] += ps.nt[x];
      if (ps.nt[x] > 0) ++itc[x];
    }
    ld_base += 2 * n;
  }
  tc_commit(bar0 + 8 * C::B_DRAIN);
  mbar_drain(bar0 + 8 * C::B_DRAIN, 0);
}

// Softmax, correction and epilogue of one stage (warps 4x .. 4x + 3; thread r
// owns query row r of the stage's block, TMEM lane r).  O is rescaled after
// P is stored (fewer live registers); P_X(j-1) V(j-1) has completed by then
// because S_X(j), whose completion was awaited, was issued after it.
template <int D>
__device__ __forceinline__ void pair_softmax(const AttnParams& p, uint32_t sQ, uint32_t sKV,
                                             uint32_t bar0, uint32_t tmem, int n_items,
                                             volatile int* abort) {
  using C = PairCfg<D>;
  constexpr int BN = C::BN;
  const int x = threadIdx.x >> 7;
  const int r = threadIdx.x & 127;
  const int warp = r >> 5, lane = threadIdx.x & 31;
  const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const uint32_t s_col = C::S_COL + x * BN, o_col = C::O_COL + x * D;
  const uint32_t sfull = bar0 + 8 * (C::B_SFULL + x), pfull = bar0 + 8 * (C::B_PFULL + x);
  const int G = p.G;
  uint32_t g = 0, ld_base = 0, q_cnt = 0;
  bool ok = true;
  ItemStream items(p.items, n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const PairShape ps = pair_shape(w, p.tpb, BN);
    const int n = ps.n, tok = ps.tok[x], nt = ps.nt[x];
    if (n == 0 && tok == 0) continue;
    const int n_rows = tok * G;
    const bool real = r < n_rows;
    const bool warp_active = warp * 32 < n_rows;
    const int q_first = w.q_tok0 + x * p.tpb;
    const int t = w.t_base + q_first + r / G;
    const int h = w.kvh * G + r % G;
    if (n > 0) {
      // Q: copy this stage's rows from the staging buffer into TMEM (bf16
      // pairs, element 2c in the low half of column c, as the MMA reads A),
      // then release the staging buffer.  Every softmax warp arrives, so the
      // release completes only after both stages copied.
      if (!warp_wait(bar0 + 8 * C::B_QFULL, q_cnt & 1, abort)) { ok = false; break; }
      if (nt > 0 && warp_active) {
        const uint32_t src = sQ + x * C::Q_BYTES + r * 128;
#pragma unroll
        for (int h32 = 0; h32 < D / 64; ++h32) {
          uint32_t qv[32];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t a = src + h32 * C::Q_CHUNK + ((u ^ (r & 7)) << 4);
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(qv[4 * u]), "=r"(qv[4 * u + 1]), "=r"(qv[4 * u + 2]),
                           "=r"(qv[4 * u + 3])
                         : "r"(a));
          }
          tmem_st32(trow + C::Q_COL + x * (D / 2) + h32 * 32, qv);
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar0 + 8 * C::B_QSMEM);
        if (nt > 0) mbar_arrive(bar0 + 8 * (C::B_QTMEM + x));
      }
      ++q_cnt;
    }
    if (tok > 0 && nt == 0) {
      // no key is visible to any row of this stage: O = 0, LSE = -inf
      if (real) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)t * p.Hq + h) * D);
        for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
        if (p.lse) p.lse[(size_t)t * p.Hq + h] = -INFINITY;
      }
    }
    if (nt == 0) {
      ld_base += 2 * n;
      continue;
    }
    const int i_r = q_first + r / G;
    const int lim = min(ps.lim[x], i_r + (w.kv_len - w.q_len) + 1);
    // the stage whose P V first reads the last tile cleans its V rows past kv_len
    const bool zero_v = ((n - 1) * BN + BN > w.kv_len) &&
                        ((x == 0 && ps.nt[0] == n) || (x == 1 && ps.nt[0] < n));
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = 0; j < nt && ok; ++j) {
      if (!warp_wait(sfull, g & 1, abort)) { ok = false; break; }
      tc_fence_after();
      const int n0 = j * BN;
      if (warp_active) {
        float sc[BN];
        {
          uint32_t v[BN / 32][32];
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) tmem_ld32(trow + s_col + c * 32, v[c]);
          tmem_ld_wait(v[0]);
#pragma unroll
          for (int c = 1; c < BN / 32; ++c) reg_tie(v[c]);
#pragma unroll
          for (int c = 0; c < BN / 32; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) sc[c * 32 + e] = __uint_as_float(v[c][e]);
        }
        const int nvis = lim - n0;
        if (nvis < BN) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= nvis) sc[c] = -INFINITY;   // mask by select, never by add
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < BN; ++c) mx = fmaxf(mx, sc[c]);
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        const bool need = real && (m_new > m_run + kRescaleThreshold);
        const bool rescale_warp = j > 0 && __any_sync(0xffffffffu, need && m_run != -INFINITY);
        const float alpha = need ? ex2_approx(m_run - m_new) : 1.0f;
        if (need) {
          l_run *= alpha;
          m_run = m_new;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        float rowsum = 0.f;
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float p0 = ex2_approx(fmaf(sc[c * 32 + e], p.scale_log2, -m_use));
            const float p1 = ex2_approx(fmaf(sc[c * 32 + e + 1], p.scale_log2, -m_use));
            rowsum += p0 + p1;
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
          // P overwrites the first BN/2 columns of this stage's S buffer
          tmem_st16(trow + s_col + c * 16, pk);
        }
        l_run += rowsum;
        if (rescale_warp) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(trow + o_col + c * 32, v);
            tmem_ld_wait(v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st32(trow + o_col + c * 32, v);
          }
        }
        tmem_st_wait();
      }
      if (j == n - 1 && zero_v) {
        // rows at and past kv_len of the last V tile: tail slots or rows never
        // loaded; P is 0 there but 0 * NaN would still poison O
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull);
      ++g;
    }
    if (!ok) break;
    // ---- epilogue: O / l -> out, LSE
    if (!warp_wait(bar0 + 8 * (C::B_PVDONE + x), (g - 1) & 1, abort)) { ok = false; break; }
    tc_fence_after();
    if (warp_active) {
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      const float lse_v = l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + o_col + c * 32, v);
        tmem_ld_wait(v);
        if (real) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)t * p.Hq + h) * D + c * 32);
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
      if (real && p.lse) p.lse[(size_t)t * p.Hq + h] = lse_v;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar0 + 8 * (C::B_OEMPTY + x));
    ld_base += 2 * n;
  }
}

template <int D>
__global__ void __maxnreg__(168)
    pa_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = PairCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sQ = base;
  const uint32_t sKV = base + 2 * C::Q_BYTES;
  const uint32_t bar0 = sKV + C::NSLOT * C::SLOT_BYTES;
  uint8_t* bar_ptr = smem + 2 * C::Q_BYTES + C::NSLOT * C::SLOT_BYTES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ptr + 8 * C::NBAR);
  volatile int* abort = reinterpret_cast<volatile int*>(bar_ptr + 8 * C::NBAR + 4);

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(bar0 + 8 * C::B_QFULL, 1);
    mbar_init(bar0 + 8 * C::B_QSMEM, 8);
    mbar_init(bar0 + 8 * (C::B_QTMEM + 0), 4);
    mbar_init(bar0 + 8 * (C::B_QTMEM + 1), 4);
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(bar0 + 8 * (C::B_KVFULL + i), 1);
      mbar_init(bar0 + 8 * (C::B_KVEMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar0 + 8 * (C::B_SFULL + i), 1);
      mbar_init(bar0 + 8 * (C::B_PFULL + i), 4);
      mbar_init(bar0 + 8 * (C::B_PVDONE + i), 1);
      mbar_init(bar0 + 8 * (C::B_OEMPTY + i), 4);
    }
    mbar_init(bar0 + 8 * C::B_DRAIN, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::PRODUCER_WARP && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == C::Q_WARP && (threadIdx.x & 31) == 0) tma_prefetch_desc(&tm_q);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int n_items = p.hdr->n_items2;

  if (warp == C::PRODUCER_WARP) {
    pair_producer<D>(&tm_k, &tm_v, p, sKV, bar0, n_items, abort);
  } else if (warp == C::Q_WARP) {
    pair_q_loader<D>(&tm_q, p, sQ, bar0, n_items, abort);
  } else if (warp == C::MMA_WARP) {
    if ((threadIdx.x & 31) == 0) pair_mma<D>(p, sKV, bar0, tmem, n_items, abort);
    __syncwarp();
  } else {
    pair_softmax<D>(p, sQ, sKV, bar0, tmem, n_items, abort);
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(p.status, kStatusTimeout);
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace pa
