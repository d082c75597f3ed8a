// pa_decode.cuh -- decode attention with keys on the MMA's M side (sm_100a,
// head_dim 128/256, G <= 32 query heads per KV head, one query token per request).
//
// In decode a (request, KV head) pair has only G query rows (G = Hq / Hkv),
// so a 128-row query tile would spend 128/G times the useful tensor work and
// the power that goes with it.  Here the products are transposed so that the
// 128 keys of a tile fill the MMA's M dimension and the G rows (padded to NR =
// 16 or 32) are its N dimension:
//   S^T = K Q^T          M = 128 keys, N = NR rows, K = D   (A = K tile, B = Q)
//   O^T += V^T P^T       M = 128 of D, N = NR rows, K = 128 keys
//                        (A = V tile read MN-major, B = P^T written by softmax)
// The online softmax of "FlashAttention" (Dao et al., Algorithm 1) then runs
// across threads: thread t owns key t of the tile (TMEM lane t of S^T) and
// d = t of every 128-wide half of O^T.  Row maxima are block reductions per
// tile; row sums stay per thread and are reduced once in the epilogue, which
// is exact because every thread rescales its partial sum by the same factor.
//
// Roles (8 warps, one CTA per SM):
//   warps 0-3  softmax / correction / epilogue
//   warps 4, 7 K/V producers (page-table-driven TMA, order K0 K1 V0 K2 V1 ...);
//              warp 4 issues the even loads of that order, warp 7 the odd ones:
//              one issuing warp per SM does not keep HBM busy with page-sized boxes
//   warp  5    MMA issuer (warp-collective issue)
//   warp  6    Q loader (Q tiles of NR rows, double-buffered where room allows)
//
// E4M3 pools (F8): the producers' TMA boxes land in a ring of fp8 staging
// tiles (128-byte swizzled rows); four more warps (8-11) widen each tile to
// fp16 (every E4M3 value is exact in fp16).  A K tile is widened straight into
// tensor memory, thread t writing key t's row into TMEM lane t, and S^T takes
// its A operand from there; a V tile is widened into the swizzled shared-memory
// slot the O^T product reads MN-major, with the rows past the request's end
// zeroed.  Shared-memory traffic per key is then the fp8 tile written and read
// once plus one fp16 V row written and read once.  The products run as fp16
// MMAs: Q is rounded to fp16 by the Q loader and P is written as fp16.  The K descale multiplies
// the softmax scale and the V descale the epilogue's 1 / l, so the pools are
// never dequantised in memory (the fp8-descale variants with a bf16 output of
// "[Perf][FA4] Warm up dense (paged) FA4 attention kernels", vLLM PR #48156,
// Summary and the review thread on the per-arch selector).
#pragma once

#include "pa_kernels.cuh"

namespace pa {

template <int D, int NR, bool F8 = false>
struct DecCfg {
  static_assert(D == 128 || D == 256, "decode kernel: head_dim 128 or 256");
  static_assert(NR == 16 || NR == 32, "decode kernel: 16 or 32 padded rows");
  static constexpr int BN = 128;                      // keys per tile (M of S^T)
  static constexpr int DCH = D / 64;                  // 128-byte column chunks of a K/V row
  static constexpr int DH = D / 128;                  // M = 128 halves of O^T
  static constexpr int SLOT_CHUNK = BN * 128;         // one 64-column chunk of a K/V tile
  static constexpr int SLOT_BYTES = BN * D * 2;       // 16-bit K/V tile the MMA reads
  // 16-bit K/V slots; with E4M3 pools V slots only, plus NST fp8 staging
  // tiles (D / 128 chunks of BN rows x 128 bytes, 128-byte swizzle)
  static constexpr int NSLOT = !F8 ? ((D == 128) ? 6 : 3) : ((D == 128) ? (NR == 16 ? 4 : 3) : 2);
  static constexpr int NST = !F8 ? 0 : ((D == 128) ? (NR == 16 ? 5 : 6) : 2);
  static constexpr int STAGE_BYTES = BN * D;
  static constexpr int Q_CHUNK = NR * 128;            // Q tile: NR rows x 64 columns per chunk
  static constexpr int Q_BYTES = NR * D * 2;
  static constexpr int QBUF = (D == 256 && NR == 32) ? 1 : 2;   // Q tiles in flight
  static constexpr int P_CHUNK = NR * 128;            // P^T: NR rows x 64 keys per chunk
  static constexpr int P_BYTES = NR * BN * 2;
  static constexpr int RED_BYTES = 3 * 4 * NR * 4;    // row maxima of 4 warps (two tiles), row sums
  static constexpr int S_COL = 0;                     // + buffer * NR
  static constexpr int O_COL = 2 * NR;                // + half * NR
  // widened K tiles (F8): NKB buffers of D / 2 columns (fp16 pairs), A of S^T
  static constexpr int NKB = (D == 128) ? 4 : 2;
  static constexpr int K_COL = D;
  static constexpr int TMEM_USED = F8 ? K_COL + NKB * D / 2 : O_COL + DH * NR;
  static constexpr int TMEM_COLS =
      TMEM_USED <= 32 ? 32 : (TMEM_USED <= 64 ? 64 : (TMEM_USED <= 128 ? 128 : (TMEM_USED <= 256 ? 256 : 512)));
  static constexpr int THREADS = F8 ? 384 : 256;
  // E4M3 variant: launched with LAUNCH_REGS per thread (384 threads, one CTA
  // per SM); the softmax warpgroup then takes SOFTMAX_REGS (up to 32 rows of
  // running maxima, sums, scores and scale factors per thread), the producer /
  // MMA / Q warpgroup and the widening warpgroup give registers back.  The
  // budgets sum to at most the launch pool (the host checks the compiled
  // launch count before any launch).
  static constexpr int LAUNCH_REGS = 168;
  static constexpr int SOFTMAX_REGS = 224, WG1_REGS = 80, CONV_REGS = 128;
  static_assert(!F8 || 128 * (SOFTMAX_REGS + WG1_REGS + CONV_REGS) <= THREADS * LAUNCH_REGS,
                "warpgroup register budgets exceed the launch pool");
  static constexpr int PRODUCER_WARP = 4, MMA_WARP = 5, Q_WARP = 6, PRODUCER2_WARP = 7;
  static constexpr int CONV_WARP0 = 8;                // E4M3 widening warps 8-11
  // barriers: q_full[2], q_empty[2], kv_full[NSLOT], kv_empty[NSLOT], s_full[2],
  //           p_full[2], pv_done[2], o_empty, drain, red[2] (row maxima), red_sum,
  //           st_full[NST], st_empty[NST] (fp8 staging), k_full[NKB], k_empty[NKB]
  //           (widened K in TMEM); with F8 kv_full / kv_empty guard the V slots
  static constexpr int B_QFULL = 0, B_QEMPTY = 2, B_KVFULL = 4, B_KVEMPTY = 4 + NSLOT,
                       B_SFULL = 4 + 2 * NSLOT, B_PFULL = B_SFULL + 2, B_PVDONE = B_PFULL + 2,
                       B_OEMPTY = B_PVDONE + 2, B_DRAIN = B_OEMPTY + 1, B_RED = B_DRAIN + 1,
                       B_REDSUM = B_RED + 2, B_STFULL = B_REDSUM + 1, B_STEMPTY = B_STFULL + NST,
                       B_KFULL = B_STEMPTY + NST, B_KEMPTY = B_KFULL + NKB,
                       B_MERGE = B_KFULL + (F8 ? 2 * NKB : 0), NBAR = B_MERGE + 1;
  static constexpr int BAR_BYTES = F8 ? 384 : 256;
  static constexpr int SMEM_BYTES = 1024 + NSLOT * SLOT_BYTES + NST * STAGE_BYTES +
                                    QBUF * Q_BYTES + 2 * P_BYTES + RED_BYTES + BAR_BYTES;
  static_assert(NBAR * 8 + 16 <= BAR_BYTES, "barrier area");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(TMEM_USED <= TMEM_COLS, "TMEM columns");
};

// Q loader: the NR-row Q tile of each item (rows past G * n_tok are left as
// they are; they only feed columns of S^T and O^T that are never read).  For
// E4M3 pools the tile is rounded to fp16 (the MMA's A and B share one type).
template <int D, int NR, bool F8>
__device__ __forceinline__ void dec_q_loader(const AttnParams& p, uint32_t sQ, uint32_t bar0,
                                             int n_items, volatile int* abort) {
  using C = DecCfg<D, NR, F8>;
  const int lane = threadIdx.x & 31;
  const int G = p.G;
  uint32_t q_cnt = 0;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (items.next(w)) {
    if (w.kv_hi <= w.kv_lo) continue;
    const uint32_t qb = q_cnt % C::QBUF;
    if (!warp_wait(bar0 + 8 * (C::B_QEMPTY + qb), ((q_cnt / C::QBUF) & 1) ^ 1, abort)) break;
    const uint32_t base = sQ + qb * C::Q_BYTES;
    const int rows = w.n_tok * G;
    const int units = rows * (D / 8);                 // 16-byte pieces
    const int t0 = w.t_base + w.q_tok0;
    for (int u0 = 0; u0 < units; u0 += 4 * 32) {
      uint4 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int u = u0 + k * 32 + lane;
        if (u < units) {
          const int r = u / (D / 8), c16 = u % (D / 8);
          const int t = t0 + r / G, h = w.kvh * G + r % G;
          v[k] = __ldg(reinterpret_cast<const uint4*>(p.q + ((size_t)t * p.Hq + h) * D) + c16);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int u = u0 + k * 32 + lane;
        if (u < units) {
          const int r = u / (D / 8), c16 = u % (D / 8);
          const uint32_t dst =
              base + (c16 >> 3) * C::Q_CHUNK + r * 128 + (((c16 & 7) ^ (r & 7)) << 4);
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
    if (lane == 0) mbar_arrive(bar0 + 8 * (C::B_QFULL + qb));
    ++q_cnt;
  }
}

// K/V producer: tiles of 128 keys in kv_sequence order; one TMA box per page
// (or part of a page) per 128-byte column chunk, lane k issuing box k.
// Producer `which` (0 or 1) issues the loads whose index has that parity and
// skips the others.  Each lane reads its page id from the table right before
// its box: a scheme that loaded ids three tiles ahead and rotated them through
// registers ran the decode step 12 % slower (bf16) and 25 % slower (E4M3),
// since every producer then walked and waited on every load's table read.
// With E4M3 pools the boxes go to the fp8 staging ring at `sKV` instead of the
// 16-bit slots.
template <int D, int NR, bool F8>
__device__ __forceinline__ void dec_producer(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                             const AttnParams& p, uint32_t sKV, uint32_t bar0,
                                             int n_items, uint32_t which, volatile int* abort) {
  using C = DecCfg<D, NR, F8>;
  constexpr int RING = F8 ? C::NST : C::NSLOT;
  constexpr int B_FULL = F8 ? C::B_STFULL : C::B_KVFULL;
  constexpr int B_EMPTY = F8 ? C::B_STEMPTY : C::B_KVEMPTY;
  constexpr int RING_BYTES = F8 ? C::STAGE_BYTES : C::SLOT_BYTES;
  constexpr int NCH = F8 ? D / 128 : C::DCH;  // boxes (128-byte column chunks) per page part
  constexpr int CH_ELEMS = F8 ? 128 : 64;     // elements of one chunk
  const int lane = threadIdx.x & 31;
  uint32_t ld_idx = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const int n = item_tiles(w, C::BN);
    for (int s = 0; s < 2 * n; ++s, ++ld_idx) {
      if ((ld_idx & 1u) != which) continue;
      int j;
      bool is_v;
      kv_sequence(s, n, j, is_v);
      const uint32_t slot = ld_idx % RING;
      if (!warp_wait(bar0 + 8 * (B_EMPTY + slot), ((ld_idx / RING) & 1) ^ 1, abort)) {
        ok = false;
        break;
      }
      const int n0 = w.kv_lo + j * C::BN;
      // every live row of the tile is loaded (rows past the item's range
      // included) so that no stale shared memory meets the products
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
          tma_load_4d(dst + c * C::SLOT_CHUNK, tm, full, c * CH_ELEMS, w.kvh, r & (p.ps - 1), page);
      }
    }
  }
  if (!ok || *abort) {
    // wait (bounded) for this producer's copies still in flight
    if (lane == 0) {
      const uint32_t first = ld_idx > (uint32_t)RING ? ld_idx - RING : 0;
      for (uint32_t k = first; k < ld_idx; ++k)
        if ((k & 1u) == which) mbar_drain(bar0 + 8 * (B_FULL + k % RING), (k / RING) & 1);
    }
  }
}

// E4M3 widening (warps 8-11, 128 threads).  Walks the producers' load order;
// staging tile i % NST holds load i as D / 128 chunks of 128 rows x 128 bytes,
// 16-byte unit x of row r stored at x ^ (r & 7) (the TMA 128-byte swizzle).
//   K tile of tile g: thread t widens key t's row and stores it to TMEM lane
//     t, columns K_COL + (g % NKB) * D / 2 onwards (fp16 pairs, element 2c in the
//     low half of column c); reading unit x of rows t..t+7 hits 8 distinct
//     bank groups thanks to the swizzle.
//   V tile of tile g: 16-bit slot g % NSLOT; the 8 lanes of a phase take one
//     16-byte unit of 8 consecutive rows, whose swizzled places (staging and
//     slot alike) fall in 8 distinct bank groups, and write its 16 halves as
//     two 16-byte units of the slot's swizzled rows.  Rows at and past the
//     request's end are written as zeros (P is 0 there, but 0 * NaN is not).
template <int D, int NR>
__device__ __forceinline__ void dec_convert(const AttnParams& p, uint32_t sKV, uint32_t sST,
                                            uint32_t bar0, uint32_t tmem, int n_items,
                                            volatile int* abort) {
  using C = DecCfg<D, NR, true>;
  constexpr int UPR = D / 16;                        // 16-byte fp8 units per row
  constexpr int UNITS = C::BN * UPR;
  const int ct = threadIdx.x - 32 * C::CONV_WARP0;   // 0..127
  const int lane = threadIdx.x & 31;
  // this warp's TMEM lanes (warp 8 + i owns lanes 32 i .. 32 i + 31)
  const uint32_t tl = tmem + (static_cast<uint32_t>((ct >> 5) * 32) << 16);
  uint32_t ld_idx = 0, g = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const int n = item_tiles(w, C::BN);
    for (int s = 0; s < 2 * n; ++s) {
      int j;
      bool is_v;
      kv_sequence(s, n, j, is_v);
      const uint32_t st = ld_idx % C::NST, tile = g + j;
      if (!warp_wait(bar0 + 8 * (C::B_STFULL + st), (ld_idx / C::NST) & 1, abort)) {
        ok = false;
        break;
      }
      const uint32_t src0 = sST + st * C::STAGE_BYTES;
      if (!is_v) {
        const uint32_t kb = tile % C::NKB;
        if (!warp_wait(bar0 + 8 * (C::B_KEMPTY + kb), ((tile / C::NKB) & 1) ^ 1, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t row_src = src0 + ct * 128;
        const uint32_t col0 = tl + C::K_COL + kb * (D / 2);
        // all of the row's loads first (8 units per pass), then widen and store
#pragma unroll
        for (int k0 = 0; k0 < UPR; k0 += 8) {
          uint32_t x[8][4];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int k = k0 + e;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(x[e][0]), "=r"(x[e][1]), "=r"(x[e][2]), "=r"(x[e][3])
                         : "r"(row_src + (k >> 3) * C::SLOT_CHUNK + (((k & 7) ^ (ct & 7)) << 4)));
          }
#pragma unroll
          for (int e2 = 0; e2 < 8; e2 += 2) {
            uint32_t h[16];
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
              for (int q = 0; q < 4; ++q)
                e4m3x4_to_f16x4(x[e2 + e][q], h[8 * e + 2 * q], h[8 * e + 2 * q + 1]);
            tmem_st16(col0 + (k0 + e2) * 8, h);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar0 + 8 * (C::B_KFULL + kb));
          mbar_arrive(bar0 + 8 * (C::B_STEMPTY + st));
        }
      } else {
        const uint32_t slot = tile % C::NSLOT;
        if (!warp_wait(bar0 + 8 * (C::B_KVEMPTY + slot), ((tile / C::NSLOT) & 1) ^ 1, abort)) {
          ok = false;
          break;
        }
        const int n0 = w.kv_lo + j * C::BN;
        const int zero_from = max(0, min(C::BN, w.kv_len - n0));
        const uint32_t dst0 = sKV + slot * C::SLOT_BYTES;
        // 8 units per pass: every load of the pass before any store.  Unit u
        // is row (u & 7) + 8 (u / (8 UPR)), column unit (u / 8) % UPR: the 8
        // lanes of a phase take 8 consecutive rows at one unit, so both the
        // swizzled staging loads and the swizzled fp16 stores hit 8 distinct
        // bank groups
#pragma unroll
        for (int u0 = 0; u0 < UNITS; u0 += 8 * 128) {
          uint32_t x[8][4];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int u = u0 + e * 128 + ct;
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
            const int u = u0 + e * 128 + ct;
            const int row = (u & 7) + 8 * (u / (8 * UPR)), k = (u >> 3) % UPR;
            uint32_t h[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) e4m3x4_to_f16x4(x[e][q], h[2 * q], h[2 * q + 1]);
            // halves 0-7 go to 16-byte unit 2 (k & 3) of the 64-column chunk
            // k / 4, halves 8-15 to the next unit (x stored at x ^ (row & 7))
            const uint32_t rbase = dst0 + (k >> 2) * C::SLOT_CHUNK + row * 128;
            const uint32_t x0 = 2 * (k & 3);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             rbase + ((x0 ^ (row & 7)) << 4)),
                         "r"(h[0]), "r"(h[1]), "r"(h[2]), "r"(h[3])
                         : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             rbase + (((x0 + 1) ^ (row & 7)) << 4)),
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
      ++ld_idx;
    }
    g += n;
  }
}

// Compensated O^T product of a request with fewer than kCompKeys keys (one
// tile, keys kCompKeys .. BN - 1 masked): the softmax stored P_lo^T, the
// rounding remainder of the 16-bit P^T of key t, at key position t + 64 of
// the P^T buffer (the second 64-key chunk, unused by such a tile).  The
// regular product already multiplied that chunk by V rows 64 .. 127, which are
// zeros past the request's end; this adds V rows 0 .. 63 times P_lo^T.
template <int D, int NR>
__device__ __forceinline__ void dec_issue_o_lo(uint32_t tmem, uint32_t slot_addr, uint32_t pb,
                                               uint32_t idesc) {
  using C = DecCfg<D, NR>;
  static_assert(kCompKeys == 64 && C::BN == 128, "P_lo^T uses the second 64-key chunk");
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint64_t bd = smem_desc_sw128(pb + C::P_CHUNK + kk * 32, 16, 1024);
#pragma unroll
    for (int hh = 0; hh < C::DH; ++hh) {
      const uint64_t ad = smem_desc_sw128(slot_addr + 2 * hh * C::SLOT_CHUNK + kk * 16 * 128,
                                          C::SLOT_CHUNK, 1024);
      mma_ss_w(tmem + C::O_COL + hh * NR, ad, bd, idesc, 1u);
    }
  }
}

// MMA issuer (all 32 lanes; one elected lane issues).  Per item of n tiles:
//   S^T(0) | S^T(1) O^T+=V(0)^T P^T(0) | S^T(2) O^T+=V(1)^T P^T(1) | ...
// g counts tiles over all items: S^T(g) and P^T(g) use buffer g & 1.
template <int D, int NR>
__device__ __forceinline__ void dec_mma(const AttnParams& p, uint32_t sQ, uint32_t sKV,
                                        uint32_t sP, uint32_t bar0, uint32_t tmem, int n_items,
                                        volatile int* abort) {
  using C = DecCfg<D, NR>;
  constexpr uint32_t kIdescS = idesc_bf16_f32(128, NR, false, false);
  constexpr uint32_t kIdescO = idesc_bf16_f32(128, NR, true, false);
  uint32_t ld_idx = 0, g = 0, q_cnt = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;

  auto kv_wait = [&](uint32_t idx) -> bool {
    const uint32_t slot = idx % C::NSLOT;
    if (!warp_wait(bar0 + 8 * (C::B_KVFULL + slot), (idx / C::NSLOT) & 1, abort)) return false;
    tc_fence_after();
    return true;
  };
  // S^T(gs) = K Q^T: A = K tile (K-major, 128 keys), B = Q tile (K-major, NR rows)
  auto issue_s = [&](uint32_t gs, uint32_t k_idx, uint32_t sQb) {
    const uint32_t slot_addr = sKV + (k_idx % C::NSLOT) * C::SLOT_BYTES;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t ad =
          smem_desc_sw128(slot_addr + (kk >> 2) * C::SLOT_CHUNK + (kk & 3) * 32, 16, 1024);
      const uint64_t bd = smem_desc_sw128(sQb + (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32, 16, 1024);
      mma_ss_w(tmem + C::S_COL + (gs & 1) * NR, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
    }
    tc_commit_w(bar0 + 8 * (C::B_SFULL + (gs & 1)));
  };
  // O^T += V^T P^T(gp): A = V tile read MN-major (M = 128 columns of D),
  // B = P^T (K-major, NR rows x 128 keys)
  auto issue_o = [&](uint32_t gp, uint32_t v_idx, bool first, bool comp) {
    const uint32_t slot_addr = sKV + (v_idx % C::NSLOT) * C::SLOT_BYTES;
    const uint32_t pb = sP + (gp & 1) * C::P_BYTES;
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk) {
      const uint64_t bd = smem_desc_sw128(pb + (kk >> 2) * C::P_CHUNK + (kk & 3) * 32, 16, 1024);
#pragma unroll
      for (int hh = 0; hh < C::DH; ++hh) {
        const uint64_t ad = smem_desc_sw128(slot_addr + 2 * hh * C::SLOT_CHUNK + kk * 16 * 128,
                                            C::SLOT_CHUNK, 1024);
        mma_ss_w(tmem + C::O_COL + hh * NR, ad, bd, kIdescO, (!first || kk > 0) ? 1u : 0u);
      }
    }
    if (comp) dec_issue_o_lo<D, NR>(tmem, slot_addr, pb, kIdescO);
    tc_commit_w(bar0 + 8 * (C::B_PVDONE + (gp & 1)));
  };

  while (ok && items.next(w)) {
    const int n = item_tiles(w, C::BN);
    if (n == 0) continue;
    const uint32_t qb = q_cnt % C::QBUF;
    const uint32_t sQb = sQ + qb * C::Q_BYTES;
    if (!warp_wait(bar0 + 8 * (C::B_QFULL + qb), (q_cnt / C::QBUF) & 1, abort)) { ok = false; break; }
    tc_fence_after();
    if (!kv_wait(ld_idx)) { ok = false; break; }
    issue_s(g, ld_idx, sQb);
    tc_commit_w(bar0 + 8 * (C::B_KVEMPTY + ld_idx % C::NSLOT));
    if (n == 1) tc_commit_w(bar0 + 8 * (C::B_QEMPTY + qb));
    for (int j = 0; j < n && ok; ++j) {
      if (j + 1 < n) {
        const uint32_t k_idx = ld_idx + (2 * (j + 1) - 1);
        if (!kv_wait(k_idx)) { ok = false; break; }
        issue_s(g + j + 1, k_idx, sQb);
        tc_commit_w(bar0 + 8 * (C::B_KVEMPTY + k_idx % C::NSLOT));
        if (j + 2 == n) tc_commit_w(bar0 + 8 * (C::B_QEMPTY + qb));
      }
      const uint32_t v_idx = ld_idx + (j == n - 1 ? 2 * n - 1 : 2 * j + 2);
      if (!kv_wait(v_idx)) { ok = false; break; }
      const uint32_t gp = g + j;
      if (!warp_wait(bar0 + 8 * (C::B_PFULL + (gp & 1)), (gp >> 1) & 1, abort)) { ok = false; break; }
      if (j == 0 && !warp_wait(bar0 + 8 * C::B_OEMPTY, (q_cnt & 1) ^ 1, abort)) { ok = false; break; }
      tc_fence_after();
      issue_o(gp, v_idx, j == 0, w.kv_len < kCompKeys);
      tc_commit_w(bar0 + 8 * (C::B_KVEMPTY + v_idx % C::NSLOT));
    }
    g += n;
    ld_idx += 2 * n;
    ++q_cnt;
  }
  tc_commit_w(bar0 + 8 * C::B_DRAIN);
  if ((threadIdx.x & 31) == 0) mbar_drain(bar0 + 8 * C::B_DRAIN, 0);
  __syncwarp();
}

// MMA issuer for E4M3 pools: the same order as dec_mma, with S^T's A operand
// (the widened K tile of tile g) read from TMEM buffer g % NKB and the V tile of
// tile g from 16-bit slot g % NSLOT; fp16 operands.
template <int D, int NR>
__device__ __forceinline__ void dec_mma_f8(const AttnParams& p, uint32_t sQ, uint32_t sKV,
                                           uint32_t sP, uint32_t bar0, uint32_t tmem,
                                           int n_items, volatile int* abort) {
  using C = DecCfg<D, NR, true>;
  constexpr uint32_t kIdescS = idesc_f16_f32(128, NR, false, false);
  constexpr uint32_t kIdescO = idesc_f16_f32(128, NR, true, false);
  uint32_t g = 0, q_cnt = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;

  // S^T(gs) = K Q^T: A = widened K in TMEM (128 lanes = keys, 8 columns per
  // 16 of D), B = Q tile (K-major, NR rows)
  auto issue_s = [&](uint32_t gs, uint32_t sQb) -> bool {
    const uint32_t kb = gs % C::NKB, sb = gs & 1;
    if (!warp_wait(bar0 + 8 * (C::B_KFULL + kb), (gs / C::NKB) & 1, abort)) return false;
    tc_fence_after();
    const uint32_t a0 = tmem + C::K_COL + kb * (D / 2);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t bd = smem_desc_sw128(sQb + (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32, 16, 1024);
      mma_ts_w(tmem + C::S_COL + sb * NR, a0 + kk * 8, bd, kIdescS, kk > 0 ? 1u : 0u);
    }
    tc_commit_w(bar0 + 8 * (C::B_SFULL + sb));
    tc_commit_w(bar0 + 8 * (C::B_KEMPTY + kb));
    return true;
  };
  // O^T += V^T P^T(gp): A = V tile read MN-major, B = P^T (K-major)
  auto issue_o = [&](uint32_t gp, bool first, bool comp) -> bool {
    const uint32_t slot = gp % C::NSLOT;
    if (!warp_wait(bar0 + 8 * (C::B_KVFULL + slot), (gp / C::NSLOT) & 1, abort)) return false;
    if (!warp_wait(bar0 + 8 * (C::B_PFULL + (gp & 1)), (gp >> 1) & 1, abort)) return false;
    if (first && !warp_wait(bar0 + 8 * C::B_OEMPTY, (q_cnt & 1) ^ 1, abort)) return false;
    tc_fence_after();
    const uint32_t slot_addr = sKV + slot * C::SLOT_BYTES;
    const uint32_t pb = sP + (gp & 1) * C::P_BYTES;
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk) {
      const uint64_t bd = smem_desc_sw128(pb + (kk >> 2) * C::P_CHUNK + (kk & 3) * 32, 16, 1024);
#pragma unroll
      for (int hh = 0; hh < C::DH; ++hh) {
        const uint64_t ad = smem_desc_sw128(slot_addr + 2 * hh * C::SLOT_CHUNK + kk * 16 * 128,
                                            C::SLOT_CHUNK, 1024);
        mma_ss_w(tmem + C::O_COL + hh * NR, ad, bd, kIdescO, (!first || kk > 0) ? 1u : 0u);
      }
    }
    if (comp) dec_issue_o_lo<D, NR>(tmem, slot_addr, pb, kIdescO);
    tc_commit_w(bar0 + 8 * (C::B_PVDONE + (gp & 1)));
    tc_commit_w(bar0 + 8 * (C::B_KVEMPTY + slot));
    return true;
  };

  while (ok && items.next(w)) {
    const int n = item_tiles(w, C::BN);
    if (n == 0) continue;
    const uint32_t qb = q_cnt % C::QBUF;
    const uint32_t sQb = sQ + qb * C::Q_BYTES;
    if (!warp_wait(bar0 + 8 * (C::B_QFULL + qb), (q_cnt / C::QBUF) & 1, abort)) { ok = false; break; }
    tc_fence_after();
    if (!issue_s(g, sQb)) { ok = false; break; }
    if (n == 1) tc_commit_w(bar0 + 8 * (C::B_QEMPTY + qb));
    for (int j = 0; j < n && ok; ++j) {
      if (j + 1 < n) {
        if (!issue_s(g + j + 1, sQb)) { ok = false; break; }
        if (j + 2 == n) tc_commit_w(bar0 + 8 * (C::B_QEMPTY + qb));
      }
      if (!issue_o(g + j, j == 0, w.kv_len < kCompKeys)) { ok = false; break; }
    }
    g += n;
    ++q_cnt;
  }
  tc_commit_w(bar0 + 8 * C::B_DRAIN);
  if ((threadIdx.x & 31) == 0) mbar_drain(bar0 + 8 * C::B_DRAIN, 0);
  __syncwarp();
}

template <int NR>
__device__ __forceinline__ void ld_cols(uint32_t taddr, uint32_t (&r)[NR]);
template <>
__device__ __forceinline__ void ld_cols<16>(uint32_t taddr, uint32_t (&r)[16]) {
  tmem_ld16(taddr, r);
  tmem_ld_wait(r);
}
template <>
__device__ __forceinline__ void ld_cols<32>(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld32(taddr, r);
  tmem_ld_wait(r);
}
template <int NR>
__device__ __forceinline__ void st_cols(uint32_t taddr, const uint32_t (&r)[NR]) {
#pragma unroll
  for (int c = 0; c < NR; c += 16) tmem_st16(taddr + c, r + c);
}

// Sum (or max) of one value per thread over the 128 softmax threads for each
// of RR rows: butterfly within the warp, then the four warp results through
// shared memory behind an mbarrier (bounded wait; count 4, one arrival per warp).
template <int RR, bool MAX>
__device__ __forceinline__ bool block_reduce_rows(float (&v)[RR], float* red, uint32_t bar,
                                                  uint32_t phase, volatile int* abort) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < RR; ++r) {
    float x = v[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float y = __shfl_xor_sync(0xffffffffu, x, o);
      x = MAX ? fmaxf(x, y) : x + y;
    }
    v[r] = x;
  }
  if (lane < RR) {
    // lane r stores row r (a select chain instead of a dynamic register index)
    float x = v[0];
#pragma unroll
    for (int r = 1; r < RR; ++r) x = lane == r ? v[r] : x;
    red[warp * RR + lane] = x;
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  if (!warp_wait(bar, phase, abort)) return false;
#pragma unroll
  for (int r = 0; r < RR; ++r) {
    const float a = red[r], b = red[RR + r], c = red[2 * RR + r], d = red[3 * RR + r];
    v[r] = MAX ? fmaxf(fmaxf(a, b), fmaxf(c, d)) : (a + b) + (c + d);
  }
  return true;
}

// Softmax, correction and epilogue (warps 0-3).  Thread t owns key t of each
// tile and column d = 128 h + t of O.  Every thread holds the running maximum
// of every row (identical in all threads) and its own share of the row sums.
// A decode item is one query token: its G rows see the same keys [kv_lo, kv_hi).
// Rows G .. RR-1 (padding) are held at -inf, so their P is 0.
template <int D, int NR, int RR, bool F8>
__device__ __forceinline__ void dec_softmax(const AttnParams& p, uint32_t sKV, uint32_t sP,
                                            float* red, uint32_t bar0, uint32_t tmem,
                                            int n_items, volatile int* merge_flag,
                                            volatile int* abort) {
  using C = DecCfg<D, NR, F8>;
  constexpr int BN = C::BN;
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);   // this warp's lanes
  const int G = p.G;
  // this thread's P^T column: 16-byte unit u of row r sits at u ^ (r & 7)
  const uint32_t p_col = (t >> 6) * C::P_CHUNK + (t & 7) * 2;
  const int p_unit = (t & 63) >> 3;
  uint32_t g = 0, ld_base = 0, q_cnt = 0;
  bool ok = true;
  ItemStream items(list_items(p), n_items, p.tpb);
  WorkItem w;
  while (ok && items.next(w)) {
    const int n = item_tiles(w, BN);
    const bool split = w.n_splits > 1;
    const size_t prow0 = (((size_t)w.b * p.Hkv + w.kvh) * p.S_max + w.split) * kBM;
    const size_t orow0 = (size_t)(w.t_base + w.q_tok0) * p.Hq + (size_t)w.kvh * G;
    if (n == 0) {
      // no key: O = 0, LSE = -inf
      for (int r = 0; r < G; ++r) {
#pragma unroll
        for (int hh = 0; hh < C::DH; ++hh) {
          const int d = hh * 128 + t;
          if (split) p.part_o[(prow0 + r) * D + d] = 0.f;
          else p.out[(orow0 + r) * D + d] = 0;
        }
        if (t == 0) {
          if (split) p.part_lse[prow0 + r] = -INFINITY;
          else if (p.lse) p.lse[orow0 + r] = -INFINITY;
        }
      }
      if (split && p.fused_merge)
        split_arrive_and_merge(p, w, D, bar0 + 8 * C::B_MERGE, merge_flag, abort);
      continue;
    }
    float m_run[RR], l_part[RR];
#pragma unroll
    for (int r = 0; r < RR; ++r) {
      m_run[r] = -INFINITY;
      l_part[r] = 0.f;
    }
    for (int j = 0; j < n && ok; ++j) {
      const uint32_t gj = g + j, sb = gj & 1;
      if (!warp_wait(bar0 + 8 * (C::B_SFULL + sb), (gj >> 1) & 1, abort)) { ok = false; break; }
      tc_fence_after();
      const int n0 = w.kv_lo + j * BN;
      const bool valid = n0 + t < w.kv_hi;
      float s[RR];
      {
        uint32_t v[NR];
        ld_cols<NR>(tl + C::S_COL + sb * NR, v);
#pragma unroll
        for (int r = 0; r < RR; ++r)
          s[r] = (valid && r < G) ? __uint_as_float(v[r]) : -INFINITY;   // mask by select
      }
      float mx[RR];
#pragma unroll
      for (int r = 0; r < RR; ++r) mx[r] = s[r];
      if (!block_reduce_rows<RR, true>(mx, red + sb * 4 * RR, bar0 + 8 * (C::B_RED + sb),
                                       (gj >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      float alpha[RR];
      bool any = false;
#pragma unroll
      for (int r = 0; r < RR; ++r) {
        const float m_new = fmaxf(m_run[r], mx[r] * p.scale_log2);
        const bool need = m_new > m_run[r] + kRescaleThreshold;
        alpha[r] = need ? ex2_approx(m_run[r] - m_new) : 1.f;   // 0 while m_run is -inf
        any = any || (need && m_run[r] != -INFINITY);
        m_run[r] = need ? m_new : m_run[r];
      }
      if (any && j > 0) {
        // O^T holds the sum up to tile gj-1: wait for that product, then rescale
        const uint32_t gp = gj - 1;
        if (!warp_wait(bar0 + 8 * (C::B_PVDONE + (gp & 1)), (gp >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int hh = 0; hh < C::DH; ++hh) {
          uint32_t o[NR];
          ld_cols<NR>(tl + C::O_COL + hh * NR, o);
#pragma unroll
          for (int r = 0; r < RR; ++r) o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha[r]);
          st_cols<NR>(tl + C::O_COL + hh * NR, o);
        }
        tmem_st_wait();
      }
      // P^T[r][t] (bf16) into buffer sb: row r of the B operand of O^T.  A
      // request with fewer than kCompKeys keys also gets P_lo^T (the rounding
      // remainder) at key position t + 64, which its masked keys leave free:
      // threads t >= 64 (P = 0 there) skip their store
      const uint32_t pb = sP + sb * C::P_BYTES + p_col;
      const bool comp = w.kv_len < kCompKeys;
      if (!comp || t < kCompKeys) {
#pragma unroll
        for (int r = 0; r < RR; ++r) {
          const float m_use = m_run[r] == -INFINITY ? 0.f : m_run[r];
          const float pr = ex2_approx(fmaf(s[r], p.scale_log2, -m_use));
          l_part[r] = fmaf(l_part[r], alpha[r], pr);
          const uint32_t a = pb + r * 128 + ((p_unit ^ (r & 7)) << 4);
          const unsigned short hi = F8 ? f16_bits(pr) : bf16_bits(pr);
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(hi) : "memory");
          if (comp) {
            const float lo = pr - (F8 ? f16_to_f32(hi) : bf16_to_f32(hi));
            asm volatile("st.shared.u16 [%0], %1;" ::"r"(a + C::P_CHUNK),
                         "h"(F8 ? f16_bits(lo) : bf16_bits(lo))
                         : "memory");
          }
        }
      }
      // (with E4M3 pools the widening warps zero these rows)
      if (!F8 && j == n - 1 && n0 + BN > w.kv_len) {
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
        for (int uu = t; uu < units; uu += 128) {
          const int row = z0 + uu / (C::DCH * 8);
          const int rem = uu % (C::DCH * 8);
          const uint32_t a = base + (rem >> 3) * C::SLOT_CHUNK + row * 128 + (rem & 7) * 16;
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0) : "memory");
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar0 + 8 * (C::B_PFULL + sb));
    }
    if (!ok) break;
    g += n;
    ld_base += 2 * n;
    // ---- epilogue: O / l -> out (or the split partial), LSE
    if (!block_reduce_rows<RR, false>(l_part, red + 2 * 4 * RR, bar0 + 8 * C::B_REDSUM,
                                      q_cnt & 1, abort)) {
      ok = false;
      break;
    }
    const uint32_t gl = g - 1;
    if (!warp_wait(bar0 + 8 * (C::B_PVDONE + (gl & 1)), (gl >> 1) & 1, abort)) { ok = false; break; }
    tc_fence_after();
#pragma unroll
    for (int hh = 0; hh < C::DH; ++hh) {
      uint32_t o[NR];
      ld_cols<NR>(tl + C::O_COL + hh * NR, o);
      const int d = hh * 128 + t;
#pragma unroll
      for (int r = 0; r < RR; ++r) {
        if (r < G) {
          const float inv_l = l_part[r] > 0.f ? (F8 ? p.v_scale : 1.0f) / l_part[r] : 0.f;
          const float val = __uint_as_float(o[r]) * inv_l;
          if (split) p.part_o[(prow0 + r) * D + d] = val;
          else p.out[(orow0 + r) * D + d] = bf16_bits(val);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RR; ++r) {
      if (r < G && t == r) {
        const float lse_v =
            l_part[r] > 0.f ? (m_run[r] + log2f(l_part[r])) * 0.69314718055994531f : -INFINITY;
        if (split) p.part_lse[prow0 + r] = lse_v;
        else if (p.lse) p.lse[orow0 + r] = lse_v;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar0 + 8 * C::B_OEMPTY);
    if (split && p.fused_merge)
        split_arrive_and_merge(p, w, D, bar0 + 8 * C::B_MERGE, merge_flag, abort);
    ++q_cnt;
  }
}

// RR: registers rows per thread (G rounded up to a power of two, >= 4);
// NR: MMA rows (N), at least 16.
template <int RR>
struct DecRows {
  static_assert(RR == 4 || RR == 8 || RR == 16 || RR == 32, "decode rows");
  static constexpr int NR = RR < 16 ? 16 : RR;
};

template <int D, int RR, bool F8 = false>
__global__ void __launch_bounds__(DecCfg<D, DecRows<RR>::NR, F8>::THREADS, 1)
    __maxnreg__((F8 ? DecCfg<D, DecRows<RR>::NR, F8>::LAUNCH_REGS : 255))
    pa_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  constexpr int NR = DecRows<RR>::NR;
  using C = DecCfg<D, NR, F8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sKV = base;
  const uint32_t sST = sKV + C::NSLOT * C::SLOT_BYTES;          // fp8 staging (F8 only)
  const uint32_t sQ = sST + C::NST * C::STAGE_BYTES;
  const uint32_t sP = sQ + C::QBUF * C::Q_BYTES;
  const uint32_t off_red = C::NSLOT * C::SLOT_BYTES + C::NST * C::STAGE_BYTES +
                           C::QBUF * C::Q_BYTES + 2 * C::P_BYTES;
  float* red = reinterpret_cast<float*>(smem + off_red);
  const uint32_t bar0 = base + off_red + C::RED_BYTES;
  uint8_t* bar_ptr = smem + off_red + C::RED_BYTES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ptr + 8 * C::NBAR);
  volatile int* abort = reinterpret_cast<volatile int*>(bar_ptr + 8 * C::NBAR + 4);
  volatile int* merge_flag = reinterpret_cast<volatile int*>(bar_ptr + 8 * C::NBAR + 8);

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(bar0 + 8 * C::B_MERGE, kSoftmaxWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar0 + 8 * (C::B_QFULL + i), 1);
      mbar_init(bar0 + 8 * (C::B_QEMPTY + i), 1);
      mbar_init(bar0 + 8 * (C::B_SFULL + i), 1);
      mbar_init(bar0 + 8 * (C::B_PFULL + i), 4);
      mbar_init(bar0 + 8 * (C::B_PVDONE + i), 1);
      mbar_init(bar0 + 8 * (C::B_RED + i), 4);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      // filled by TMA (one expect_tx arrival) or by the four widening warps
      mbar_init(bar0 + 8 * (C::B_KVFULL + i), F8 ? 4 : 1);
      mbar_init(bar0 + 8 * (C::B_KVEMPTY + i), 1);
    }
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(bar0 + 8 * (C::B_STFULL + i), 1);
      mbar_init(bar0 + 8 * (C::B_STEMPTY + i), 4);
    }
    if (F8) {
      for (int i = 0; i < C::NKB; ++i) {
        mbar_init(bar0 + 8 * (C::B_KFULL + i), 4);
        mbar_init(bar0 + 8 * (C::B_KEMPTY + i), 1);
      }
    }
    mbar_init(bar0 + 8 * C::B_OEMPTY, 4);
    mbar_init(bar0 + 8 * C::B_DRAIN, 1);
    mbar_init(bar0 + 8 * C::B_REDSUM, 4);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything above overlaps the scheduler kernel; its work list is read below
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int n_items = list_count(p);

  if constexpr (F8) {
    // per-warpgroup register budgets first, then the roles
    if (warp < kSoftmaxWarps) {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::SOFTMAX_REGS));
      dec_softmax<D, NR, RR, F8>(p, sKV, sP, red, bar0, tmem, n_items, merge_flag, abort);
    } else if (warp < C::CONV_WARP0) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::WG1_REGS));
      if (warp == C::PRODUCER_WARP || warp == C::PRODUCER2_WARP)
        dec_producer<D, NR, F8>(&tm_k, &tm_v, p, sST, bar0, n_items,
                                warp == C::PRODUCER_WARP ? 0u : 1u, abort);
      else if (warp == C::Q_WARP)
        dec_q_loader<D, NR, F8>(p, sQ, bar0, n_items, abort);
      else
        dec_mma_f8<D, NR>(p, sQ, sKV, sP, bar0, tmem, n_items, abort);
    } else {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::CONV_REGS));
      dec_convert<D, NR>(p, sKV, sST, bar0, tmem, n_items, abort);
    }
  } else {
    if (warp == C::PRODUCER_WARP || warp == C::PRODUCER2_WARP) {
      dec_producer<D, NR, F8>(&tm_k, &tm_v, p, sKV, bar0, n_items,
                              warp == C::PRODUCER_WARP ? 0u : 1u, abort);
    } else if (warp == C::Q_WARP) {
      dec_q_loader<D, NR, F8>(p, sQ, bar0, n_items, abort);
    } else if (warp == C::MMA_WARP) {
      dec_mma<D, NR>(p, sQ, sKV, sP, bar0, tmem, n_items, abort);
    } else if (warp < kSoftmaxWarps) {
      dec_softmax<D, NR, RR, F8>(p, sKV, sP, red, bar0, tmem, n_items, merge_flag, abort);
    }
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
