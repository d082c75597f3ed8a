// pa_prefill.cuh -- two-stage prefill attention kernel (sm_100a, head_dim 64/128).
//
// A work item here is a PAIR of consecutive 128-row query blocks of one
// (request, KV head): stage A holds query tokens [q0, q0 + tpb), stage B the
// next tpb tokens (possibly partial or empty).  Both stages read the same K/V
// tiles, so every tile loaded feeds 256 query rows: half the K/V traffic per
// row of the one-stage kernel.  This follows the two-query-stage (q_stage = 2)
// SM100 prefill configuration that "[Perf][FA4] Warm up dense (paged) FA4
// attention kernels" (vLLM PR #48156, review thread) describes, written here
// from that description.
//
// Each stage has two S buffers in TMEM, so S_X(j+1) is computed while the
// softmax warps of stage X still work on S_X(j): per stage the softmax runs
// back to back and the tensor core fills the gaps with the other stage.  The
// MMA order per item (n tiles; stage X uses tiles j < nt[X]) is
//   S_A(0) S_B(0) | S_A(1) S_B(1) P_A(0)V(0) P_B(0)V(0) | S_A(2) S_B(2) P_A(1)V(1) ...
// so S_X(g) is always issued after P_X(g-2) V, which keeps the phases of the
// per-buffer barriers unambiguous.
//
// Roles (12 warps, one CTA per SM):
//   warps 0-3   stage A: softmax, correction, epilogue (thread r = query row r)
//   warps 4-7   the same for stage B
//   warps 8, 11 K/V producers (page-table-driven TMA; each issues the loads of
//               one parity of the order K0 K1 V0 K2 V1 ...)
//   warp  9     MMA issuer (warp-collective issue, one elected lane)
//   warp  10    Q loader (Q_A and Q_B buffers in shared memory)
// TMEM (512 columns): S_A0 S_A1 S_B0 S_B1 (BN each), O_A, O_B (D each).
// Shared memory: Q_A, Q_B, the K/V slot ring, epilogue staging, barriers.
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
  static constexpr int NSLOT = (D == 64) ? 16 : 9;
  static constexpr int EPI_WARP_BYTES = 32 * 64;       // 32 rows x 32 columns of bf16
  static constexpr int EPI_BYTES = 8 * EPI_WARP_BYTES;
  static constexpr int S_COL = 0;                      // + (2 * stage + buffer) * BN
  static constexpr int O_COL = 4 * BN;                 // + stage * D
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 384;
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, Q_WARP = 10, PRODUCER2_WARP = 11;
  // barriers: q_full[2], q_empty[2], kv_full[NSLOT], kv_empty[NSLOT],
  //           s_full[2][2], p_full[2][2], pv_done[2][2], o_empty[2], drain
  static constexpr int B_QFULL = 0, B_QEMPTY = 2, B_KVFULL = 4, B_KVEMPTY = 4 + NSLOT,
                       B_SFULL = 4 + 2 * NSLOT, B_PFULL = B_SFULL + 4, B_PVDONE = B_PFULL + 4,
                       B_OEMPTY = B_PVDONE + 4, B_DRAIN = B_OEMPTY + 2, NBAR = B_DRAIN + 1;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_BYTES =
      1024 + 2 * Q_BYTES + NSLOT * SLOT_BYTES + EPI_BYTES + BAR_BYTES;
  static_assert(NBAR * 8 + 16 <= BAR_BYTES, "barrier area");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(O_COL + 2 * D <= TMEM_COLS, "TMEM columns");
};

// Tokens of the two stages and KV tiles each needs.
struct PairShape {
  int tok[2];     // query tokens of stage A and B
  int lim[2];     // keys visible to the stage's last row (causal, end aligned)
  int nt[2];      // KV tiles of each stage (0 = the stage has nothing to do)
  int n;          // KV tiles of the item (max of the two)
};

__device__ __forceinline__ PairShape pair_shape(const WorkItem& w, int tpb, int BN, int causal) {
  PairShape s;
  s.tok[0] = max(0, min(tpb, w.q_len - w.q_tok0));
  s.tok[1] = max(0, min(tpb, w.q_len - w.q_tok0 - s.tok[0]));
  for (int x = 0; x < 2; ++x) {
    const int q0 = w.q_tok0 + x * tpb;
    int hi = causal ? q0 + s.tok[x] + (w.kv_len - w.q_len) : w.kv_len;
    hi = hi < 0 ? 0 : (hi > w.kv_len ? w.kv_len : hi);
    s.lim[x] = hi;
    s.nt[x] = s.tok[x] > 0 ? ceil_div(hi, BN) : 0;
  }
  s.n = max(s.nt[0], s.nt[1]);
  return s;
}

// Load index of K_j and V_j within an item of n tiles (the order of kv_sequence).
__device__ __forceinline__ int k_index(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int v_index(int j, int n) { return j == n - 1 ? 2 * n - 1 : 2 * j + 2; }

// Q loader: Q_X of an item goes into buffer X once the last S_X of the
// previous item that used stage X has completed (q_empty[X]).  Only stages
// with at least one tile get a Q.  Whole blocks arrive by TMA; partial blocks
// by plain loads of the live rows, stored with the TMA's 128-byte swizzle.
template <int D>
__device__ __forceinline__ void pair_q_loader(const CUtensorMap* tm_q, const AttnParams& p,
                                              uint32_t sQ, uint32_t bar0, int n_items,
                                              volatile int* abort) {
  using C = PairCfg<D>;
  const int lane = threadIdx.x & 31;
  const int G = p.G;
  const int T = p.cu_q_lens ? p.cu_q_lens[p.B] : p.B;
  uint32_t qc[2] = {0, 0};
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const PairShape ps = pair_shape(w, p.tpb, C::BN, p.causal);
    for (int x = 0; x < 2; ++x) {
      if (ps.nt[x] == 0) continue;
      if (!warp_wait(bar0 + 8 * (C::B_QEMPTY + x), (qc[x] & 1) ^ 1, abort)) { ok = false; break; }
      const uint32_t qfull = bar0 + 8 * (C::B_QFULL + x);
      const uint32_t base = sQ + x * C::Q_BYTES;
      const int t0 = w.t_base + w.q_tok0 + x * p.tpb;
      if (ps.tok[x] == p.tpb && t0 + p.tpb <= T) {
        if (lane == 0) {
          mbar_arrive_expect_tx(qfull, C::DCH * p.tpb * G * 128);
          for (int c = 0; c < C::DCH; ++c)
            tma_load_3d(base + c * C::Q_CHUNK, tm_q, qfull, c * 64, w.kvh * G, t0);
        }
      } else {
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
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(qfull);
      }
      ++qc[x];
    }
    // Q is read once, so it always comes from DRAM; pull the next item's Q
    // into L2 now so that its load at the next item boundary is short.
    WorkItem nw;
    if (ok && lane == 0 && items.peek(nw)) {
      for (int x = 0; x < 2; ++x) {
        const int t0 = nw.t_base + nw.q_tok0 + x * p.tpb;
        if (nw.q_len - nw.q_tok0 - x * p.tpb >= p.tpb && t0 + p.tpb <= T)
          for (int c = 0; c < C::DCH; ++c) tma_prefetch_l2_3d(tm_q, c * 64, nw.kvh * G, t0);
      }
    }
  }
  if (*abort && lane == 0)
    for (int x = 0; x < 2; ++x)
      if (qc[x] > 0) mbar_drain(bar0 + 8 * (C::B_QFULL + x), (qc[x] - 1) & 1);
}

// K/V producer: the tiles of an item in the MMA's consumption order
// (kv_sequence: K0 K1 V0 K2 V1 ... V(n-1)); every live row of a tile is
// loaded.  Each lane reads its page id right before its box, as in the
// one-stage producer.
template <int D>
__device__ __forceinline__ void pair_producer(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                              const AttnParams& p, uint32_t sKV, uint32_t bar0,
                                              int n_items, uint32_t which, volatile int* abort) {
  using C = PairCfg<D>;
  const int lane = threadIdx.x & 31;
  uint32_t ld_idx = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const int n = pair_shape(w, p.tpb, C::BN, p.causal).n;
    for (int s = 0; s < 2 * n; ++s, ++ld_idx) {
      if ((ld_idx & 1u) != which) continue;
      int j;
      bool is_v;
      kv_sequence(s, n, j, is_v);
      const uint32_t slot = ld_idx % C::NSLOT;
      if (!warp_wait(bar0 + 8 * (C::B_KVEMPTY + slot), ((ld_idx / C::NSLOT) & 1) ^ 1, abort)) {
        ok = false;
        break;
      }
      const int n0 = j * C::BN;
      const int live = min(w.kv_len - n0, C::BN);
      const int nbox = (live + p.box_h - 1) >> p.box_log2;
      const uint32_t full = bar0 + 8 * (C::B_KVFULL + slot);
      if (lane == 0) mbar_arrive_expect_tx(full, nbox * p.box_h * 128 * C::DCH);
      __syncwarp();
      if (lane < nbox) {
        const int r = n0 + lane * p.box_h;     // < kv_len <= C * ps
        int page = __ldg(p.page_table + (size_t)w.b * p.tstride + (r >> p.ps_log2));
        if (page < 0 || (p.num_pages > 0 && page >= p.num_pages)) {
          atomicOr(p.status, kStatusBadPage);
          page = -1;   // out of the tensor map: the box reads as zeros
        }
        const CUtensorMap* tm = is_v ? tm_v : tm_k;
        const uint32_t dst = sKV + slot * C::SLOT_BYTES + lane * p.box_h * 128;
        for (int c = 0; c < C::DCH; ++c)
          tma_load_4d(dst + c * C::SLOT_CHUNK, tm, full, c * 64, w.kvh, r & (p.ps - 1), page);
      }
    }
  }
  if (!ok || *abort) {
    if (lane == 0) {
      const uint32_t first = ld_idx > (uint32_t)C::NSLOT ? ld_idx - C::NSLOT : 0;
      for (uint32_t k = first; k < ld_idx; ++k)
        if ((k & 1u) == which) mbar_drain(bar0 + 8 * (C::B_KVFULL + k % C::NSLOT), (k / C::NSLOT) & 1);
    }
  }
}

// MMA issuer (all 32 lanes run it; one elected lane issues).  g[X] counts the
// tiles stage X has processed: S_X(g) goes to buffer g & 1, and the barriers
// of that buffer complete once per two tiles, phase (g >> 1) & 1.
template <int D>
__device__ __forceinline__ void pair_mma(const AttnParams& p, uint32_t sQ, uint32_t sKV,
                                         uint32_t bar0, uint32_t tmem, int n_items,
                                         volatile int* abort) {
  using C = PairCfg<D>;
  constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, C::BN, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, false, true);
  uint32_t ld_base = 0;
  uint32_t g[2] = {0, 0};     // tiles processed per stage
  uint32_t itc[2] = {0, 0};   // items per stage with tiles (q_full / o_empty phases)
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;

  auto kv_wait = [&](uint32_t idx) -> bool {
    const uint32_t slot = idx % C::NSLOT;
    if (!warp_wait(bar0 + 8 * (C::B_KVFULL + slot), (idx / C::NSLOT) & 1, abort)) return false;
    tc_fence_after();
    return true;
  };
  // S_X(gx) = Q_X K^T into buffer gx & 1 of stage X
  auto issue_s = [&](int x, uint32_t gx, uint32_t k_idx) {
    const uint32_t slot_addr = sKV + (k_idx % C::NSLOT) * C::SLOT_BYTES;
    const uint32_t q_addr = sQ + x * C::Q_BYTES;
    const uint32_t d_col = tmem + C::S_COL + (2 * x + (gx & 1)) * C::BN;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t ad = smem_desc_sw128(q_addr + (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32, 16, 1024);
      const uint64_t bd =
          smem_desc_sw128(slot_addr + (kk >> 2) * C::SLOT_CHUNK + (kk & 3) * 32, 16, 1024);
      mma_ss_w(d_col, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
    }
    tc_commit_w(bar0 + 8 * (C::B_SFULL + 2 * x + (gx & 1)));
  };
  // O_X += P_X(gx) V, P read from the first BN/2 columns of its S buffer
  // (compensated items: O_X += P_lo V as well, P_lo in the other BN/2 columns)
  auto issue_pv = [&](int x, uint32_t gx, uint32_t v_idx, bool first, bool comp) {
    const uint32_t slot_addr = sKV + (v_idx % C::NSLOT) * C::SLOT_BYTES;
    const uint32_t p_col = tmem + C::S_COL + (2 * x + (gx & 1)) * C::BN;
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk) {
      const uint64_t bd = smem_desc_sw128(slot_addr + kk * 16 * 128, C::SLOT_CHUNK, 1024);
      mma_ts_w(tmem + C::O_COL + x * D, p_col + kk * 8, bd, kIdescPV,
               (!first || kk > 0) ? 1u : 0u);
    }
    if (comp) {
#pragma unroll
      for (int kk = 0; kk < C::BN / 16; ++kk) {
        const uint64_t bd = smem_desc_sw128(slot_addr + kk * 16 * 128, C::SLOT_CHUNK, 1024);
        mma_ts_w(tmem + C::O_COL + x * D, p_col + C::BN / 2 + kk * 8, bd, kIdescPV, 1u);
      }
    }
    tc_commit_w(bar0 + 8 * (C::B_PVDONE + 2 * x + (gx & 1)));
  };

  while (ok && items.next(w)) {
    const PairShape ps = pair_shape(w, p.tpb, C::BN, p.causal);
    const int n = ps.n;
    if (n == 0) continue;
    const bool comp = item_compensated(w, p.causal);   // stage A's first row
    for (int x = 0; x < 2 && ok; ++x)
      if (ps.nt[x] > 0 && !warp_wait(bar0 + 8 * (C::B_QFULL + x), itc[x] & 1, abort)) ok = false;
    if (!ok) break;
    tc_fence_after();
    // tile 0: S of both stages
    if (!kv_wait(ld_base)) { ok = false; break; }
    for (int x = 0; x < 2; ++x) {
      if (ps.nt[x] == 0) continue;
      issue_s(x, g[x], ld_base);
      if (ps.nt[x] == 1) tc_commit_w(bar0 + 8 * (C::B_QEMPTY + x));
    }
    tc_commit_w(bar0 + 8 * (C::B_KVEMPTY + ld_base % C::NSLOT));
    for (int j = 0; j < n && ok; ++j) {
      if (j + 1 < n) {
        const uint32_t k_idx = ld_base + k_index(j + 1);
        if (!kv_wait(k_idx)) { ok = false; break; }
        for (int x = 0; x < 2; ++x) {
          if (j + 1 >= ps.nt[x]) continue;
          issue_s(x, g[x] + j + 1, k_idx);
          if (j + 2 == ps.nt[x]) tc_commit_w(bar0 + 8 * (C::B_QEMPTY + x));
        }
        tc_commit_w(bar0 + 8 * (C::B_KVEMPTY + k_idx % C::NSLOT));
      }
      const uint32_t v_idx = ld_base + v_index(j, n);
      if (!kv_wait(v_idx)) { ok = false; break; }
      for (int x = 0; x < 2 && ok; ++x) {
        if (j >= ps.nt[x]) continue;
        const uint32_t gx = g[x] + j;
        if (!warp_wait(bar0 + 8 * (C::B_PFULL + 2 * x + (gx & 1)), (gx >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        if (j == 0 && !warp_wait(bar0 + 8 * (C::B_OEMPTY + x), (itc[x] & 1) ^ 1, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(x, gx, v_idx, j == 0, comp);
      }
      if (!ok) break;
      tc_commit_w(bar0 + 8 * (C::B_KVEMPTY + v_idx % C::NSLOT));
    }
    for (int x = 0; x < 2; ++x) {
      g[x] += ps.nt[x];
      if (ps.nt[x] > 0) ++itc[x];
    }
    ld_base += 2 * n;
  }
  // all MMAs issued by this warp complete before TMEM is released
  tc_commit_w(bar0 + 8 * C::B_DRAIN);
  if ((threadIdx.x & 31) == 0) mbar_drain(bar0 + 8 * C::B_DRAIN, 0);
  __syncwarp();
}

// Softmax, correction and epilogue of one stage (warps 4x .. 4x + 3; thread r
// owns query row r of the stage's block, TMEM lane r).
template <int D>
__device__ __forceinline__ void pair_softmax(const CUtensorMap* tm_o, const AttnParams& p,
                                             uint32_t sKV, uint32_t sEpi, uint32_t bar0,
                                             uint32_t tmem, int n_items, volatile int* abort) {
  using C = PairCfg<D>;
  constexpr int BN = C::BN;
  const int x = threadIdx.x >> 7;
  const int r = threadIdx.x & 127;
  const int warp = r >> 5, lane = threadIdx.x & 31;
  const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const uint32_t o_col = C::O_COL + x * D;
  const int G = p.G;
  const int T = p.cu_q_lens ? __ldg(p.cu_q_lens + p.B) : p.B;
  const uint32_t sEpiW = sEpi + (4 * x + warp) * C::EPI_WARP_BYTES;
  uint32_t g = 0, ld_base = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const PairShape ps = pair_shape(w, p.tpb, BN, p.causal);
    const int n = ps.n, tok = ps.tok[x], nt = ps.nt[x];
    const bool comp = item_compensated(w, p.causal);   // stage A's first row
    const int n_rows = tok * G;
    const bool real = r < n_rows;
    const bool warp_active = warp * 32 < n_rows;
    const int q_first = w.q_tok0 + x * p.tpb;
    const int t = w.t_base + q_first + r / G;
    const int h = w.kvh * G + r % G;
    if (tok > 0 && nt == 0 && real) {
      // no key is visible to any row of this stage: O = 0, LSE = -inf
      uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)t * p.Hq + h) * D);
      for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
      if (p.lse) p.lse[(size_t)t * p.Hq + h] = -INFINITY;
    }
    if (nt == 0) {
      ld_base += 2 * n;
      continue;
    }
    const int i_r = q_first + r / G;
    const int lim = p.causal ? min(ps.lim[x], i_r + (w.kv_len - w.q_len) + 1) : ps.lim[x];
    // the stage whose P arrival gates the first P V of the last tile cleans
    // that tile's V rows at and past kv_len
    const bool zero_v = ((n - 1) * BN + BN > w.kv_len) &&
                        ((x == 0 && ps.nt[0] == n) || (x == 1 && ps.nt[0] < n));
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = 0; j < nt && ok; ++j) {
      const uint32_t gj = g + j, sb = gj & 1;
      const uint32_t s_col = C::S_COL + (2 * x + sb) * BN;
      if (!warp_wait(bar0 + 8 * (C::B_SFULL + 2 * x + sb), (gj >> 1) & 1, abort)) {
        ok = false;
        break;
      }
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
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < BN; c += 8) {
#pragma unroll
          for (int k = 0; k < 4; ++k) mx4[k] = fmax3(mx4[k], sc[c + 2 * k], sc[c + 2 * k + 1]);
        }
        const float mx = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        const bool need = real && (m_new > m_run + kRescaleThreshold);
        if (j > 0 && __any_sync(0xffffffffu, need && m_run != -INFINITY)) {
          // O holds the sum up to tile gj-1: wait for that P V, then rescale it
          const uint32_t gp = gj - 1;
          if (!warp_wait(bar0 + 8 * (C::B_PVDONE + 2 * x + (gp & 1)), (gp >> 1) & 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = need ? ex2_approx(m_run - m_new) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(trow + o_col + c * 32, v);
            tmem_ld_wait(v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st32(trow + o_col + c * 32, v);
          }
          tmem_st_wait();
        }
        if (need) {
          l_run *= ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        // s * scale_log2 - m and the row sum in packed fp32 pairs
        const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(-m_use, -m_use);
        uint64_t rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(sc[c * 32 + e], sc[c * 32 + e + 1]), sc2, nm2), x0, x1);
            const float p0 = ex2_approx(x0);
            const float p1 = ex2_approx(x1);
            rs2[(e >> 1) & 1] = f2_add(rs2[(e >> 1) & 1], f2_pack(p0, p1));
            pk[e >> 1] = pack_bf16x2(p0, p1);
            sc[c * 32 + e] = p0;
            sc[c * 32 + e + 1] = p1;
          }
          // P overwrites the first BN/2 columns of the S buffer it came from
          tmem_st16(trow + s_col + c * 16, pk);
          if (comp) {
            // P_lo = bf16(P - P_hi) into the other BN/2 columns
#pragma unroll
            for (int e = 0; e < 32; e += 2)
              pk[e >> 1] = pack_bf16x2(sc[c * 32 + e] - bf16_to_f32(pk[e >> 1] & 0xffffu),
                                       sc[c * 32 + e + 1] - bf16_to_f32(pk[e >> 1] >> 16));
            tmem_st16(trow + s_col + BN / 2 + c * 16, pk);
          }
        }
        {
          float a0, a1, b0, b1;
          f2_unpack(rs2[0], a0, a1);
          f2_unpack(rs2[1], b0, b1);
          l_run += (a0 + b0) + (a1 + b1);
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
      if (lane == 0) mbar_arrive(bar0 + 8 * (C::B_PFULL + 2 * x + sb));
    }
    if (!ok) break;
    g += nt;
    // ---- epilogue: O / l -> out, LSE
    const uint32_t gl = g - 1;
    if (!warp_wait(bar0 + 8 * (C::B_PVDONE + 2 * x + (gl & 1)), (gl >> 1) & 1, abort)) {
      ok = false;
      break;
    }
    tc_fence_after();
    if (warp_active) {
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      const float lse_v = l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      // whole blocks of 32 / G tokens per warp go out through TMA stores
      const bool o_tma = p.o_tma && tok == p.tpb && w.t_base + q_first + p.tpb <= T;
      const int t_w0 = w.t_base + q_first + warp * (32 / G);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + o_col + c * 32, v);
        tmem_ld_wait(v);
        if (o_tma) {
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
            tma_store_3d(tm_o, sEpiW, c * 32, w.kvh * G, t_w0);
            bulk_commit_group();
          }
        } else if (real) {
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
  if (lane == 0) bulk_wait_all();   // O stores complete before the CTA exits
}

template <int D>
__global__ void __maxnreg__(168)
    pa_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_o, const AttnParams p) {
  using C = PairCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sQ = base;
  const uint32_t sKV = base + 2 * C::Q_BYTES;
  const uint32_t sEpi = sKV + C::NSLOT * C::SLOT_BYTES;
  const uint32_t bar0 = sEpi + C::EPI_BYTES;
  uint8_t* bar_ptr = smem + 2 * C::Q_BYTES + C::NSLOT * C::SLOT_BYTES + C::EPI_BYTES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ptr + 8 * C::NBAR);
  volatile int* abort = reinterpret_cast<volatile int*>(bar_ptr + 8 * C::NBAR + 4);

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar0 + 8 * (C::B_QFULL + x), 1);
      mbar_init(bar0 + 8 * (C::B_QEMPTY + x), 1);
      mbar_init(bar0 + 8 * (C::B_OEMPTY + x), 4);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(bar0 + 8 * (C::B_KVFULL + i), 1);
      mbar_init(bar0 + 8 * (C::B_KVEMPTY + i), 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(bar0 + 8 * (C::B_SFULL + i), 1);
      mbar_init(bar0 + 8 * (C::B_PFULL + i), 4);
      mbar_init(bar0 + 8 * (C::B_PVDONE + i), 1);
    }
    mbar_init(bar0 + 8 * C::B_DRAIN, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if ((warp == C::PRODUCER_WARP || warp == C::PRODUCER2_WARP) && (threadIdx.x & 31) == 0) {
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

  if (warp == C::PRODUCER_WARP || warp == C::PRODUCER2_WARP) {
    pair_producer<D>(&tm_k, &tm_v, p, sKV, bar0, n_items,
                     warp == C::PRODUCER_WARP ? 0u : 1u, abort);
  } else if (warp == C::Q_WARP) {
    pair_q_loader<D>(&tm_q, p, sQ, bar0, n_items, abort);
  } else if (warp == C::MMA_WARP) {
    pair_mma<D>(p, sQ, sKV, bar0, tmem, n_items, abort);
  } else {
    pair_softmax<D>(&tm_o, p, sKV, sEpi, bar0, tmem, n_items, abort);
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
