// Tensor-core flash attention for sm_100a (full, non-causal), persistent.
//
// O = softmax(Q K^T / sqrt(dh)) V.  One CTA per SM walks work items; an item is a pair
// of 128-query tiles of one (sample row, head), handled by two softmax warpgroups.
//   warp 0    one thread streams Q (per item) and K_n / V_n^T (per key tile, two-stage
//             rings) with TMA, no multicast; each buffer is refilled as soon as the MMA
//             that read it completed (polled without blocking).
//   warp 1    allocates all 512 TMEM columns (S_0, S_1, O_0, O_1); one thread of warp 1 (group 0)
//             and one of warp 2 (group 1) each issue
//             S_g = Q_g K_n^T (M=128, N=128, K = dh padded to 80: a 128B- and a
//             32B-swizzled operand) and O_g += P_g V_n (M=128, N=DP, K=128).  The Q K^T of
//             key tile n+1 is issued before the P V of tile n, so the tensor cores run
//             while the softmax works.  Group 1 starts once group 0 has written its first P,
//             so the two groups' exp2 phases alternate on the MUFU pipe.
//   warps 4-7, 8-11  softmax of query group 0 / 1 (register budget raised with setmaxnreg,
//             taken from warpgroup 0), one query row per thread: S from TMEM
//             into registers (then S is released), online softmax in base 2 with lazy
//             O rescaling (only when the running max grows by more than 2^8), P as bf16 in
//             128B-swizzled shared memory, and at the end of an item O / l through a
//             shared-memory staging tile (the start of the group's P buffer, free once the
//             item's last P V is done) and one TMA store (O is released as soon as it is in
//             registers).  Q is double-buffered, so the next item's Q arrives while the
//             current item computes.
// Every mbarrier wait is bounded.  status[0] receives DIT_ERR_DEVICE_TIMEOUT if one runs
// out; status[1] counts the warps that moved their reference maximum (lazy rescales).
//
// Layouts: q, k [R*H, Tpad, DP] bf16 (rows of one head contiguous, head dim padded with
// zeros to DP = 80 for dh = 72); v transposed [R*H, DP, Tpad]; padded key rows are zero
// and masked to -inf in the last key tile.  o [R*T, d] bf16, token-major.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dit {

// One pair of probabilities in every kEx2PolyEvery is exponentiated with a polynomial on
// the FMA pipe (ex2_poly_f2) instead of the MUFU unit, which the exponentials and the bf16
// conversions otherwise saturate; 0 turns it off.
#ifndef DIT_EX2_POLY_EVERY
#define DIT_EX2_POLY_EVERY 4
#endif
constexpr int kEx2PolyEvery = DIT_EX2_POLY_EVERY > 0 ? DIT_EX2_POLY_EVERY : 1 << 30;

template <int DH>
struct AttnCfg {
  static constexpr int DP = (DH + 15) / 16 * 16;
  static constexpr bool TAIL = DP > 64;                 // head-dim columns 64..DP-1
  static constexpr int MAIN = 128 * 128;                // 128 rows x 64 bf16
  static constexpr int TAILB = TAIL ? 128 * 32 : 0;     // 128 rows x 16 bf16
  static constexpr int QK_TILE = MAIN + TAILB;          // one Q or K tile
  static constexpr int V_ATOM = DP * 128;               // DP rows x 64 keys
  static constexpr int V_TILE = 2 * V_ATOM;
  static constexpr int P_TILE = 2 * MAIN;               // 128 queries x 128 keys bf16
  static constexpr int O_ROW = DH * 2;                  // bytes of one output row
  static constexpr bool O_SW128 = O_ROW == 128;         // 128B-swizzled staging (else rows packed)
  static constexpr int O_TILE = (128 * O_ROW + 1023) / 1024 * 1024;
  static constexpr int Q_BUF = 2 * QK_TILE;             // Q of both query tiles of an item
  static constexpr int OFF_Q = 0;                       // two Q buffers: items alternate
  static constexpr int OFF_K = OFF_Q + 2 * Q_BUF;       // two K stages
  static constexpr int OFF_V = OFF_K + 2 * QK_TILE;     // two V^T stages
  static constexpr int OFF_P = OFF_V + 2 * V_TILE;      // P of both query tiles; each group's
                                                        // output staging tile reuses the start of
                                                        // its P buffer once the item's last P V is done
  static constexpr int OFF_BAR = OFF_P + 2 * P_TILE;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int TMEM_COLS = 512;                 // S0, S1, O0, O1 (128 columns each)
  static constexpr int THREADS = 384;                   // warpgroup 0: loads, MMA; 1, 2: softmax
  static constexpr int REG_CTRL = 96, REG_SOFTMAX = 200;
  static constexpr int REG_POOL = 128 * REG_CTRL + 256 * REG_SOFTMAX;  // must fit the launch allocation
  static_assert(QK_TILE % 1024 == 0 && V_ATOM % 1024 == 0 && OFF_P % 1024 == 0, "1024-byte aligned tiles");
  static_assert(O_ROW % 16 == 0, "16-byte output rows");
  static_assert(O_TILE <= P_TILE, "output staging inside the P buffer");
  static_assert(SMEM <= 232448, "shared memory");
};

enum {
  B_QF0 = 0, B_QF1, B_QE0, B_QE1,    // Q buffer b loaded / free (all Q K^T of its item done)
  B_KF0, B_KF1, B_KE0, B_KE1,        // K stages full / empty
  B_VF0, B_VF1, B_VE0, B_VE1,        // V^T stages full / empty
  B_S0, B_S1,                        // S_g ready
  B_SF0, B_SF1,                      // S_g read into registers (count 128)
  B_P0, B_P1,                        // P_g written (count 128)
  B_O0, B_O1,                        // P_g V done
  B_OF0, B_OF1,                      // O_g read by the epilogue (count 128)
  B_OS0, B_OS1,                      // group g's last output store has read its staging tile
  B_OW0, B_OW1,                      // output staging of group g written (count 128)
  B_GO,                              // group 0 wrote its first P: group 1 may start (completes once)
  B_COUNT
};

// Persistent flash attention.  A work item is a pair of 128-query tiles of one (sample
// row, head); CTA b walks the items b, b + gridDim.x, ...  The key tiles of all its items
// form one sequence that streams through the two-stage K / V^T rings.
template <int DH>
__global__ void __launch_bounds__(384, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQt,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKt,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO, const AttnArgs a,
                   int* status) {
  using C = AttnCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  uint32_t* holder = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * B_COUNT);
#define BAR(i) (bar0 + 8u * (i))

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (a.T + 127) / 128;            // key tiles per item
  const int nq = a.Tpad / 128;                 // query tiles per head
  const int pairs = (nq + 1) / 2;              // items per head
  const int items = a.R * a.H * pairs;
  const int my_items = static_cast<int>(blockIdx.x) < items ? (items - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int ntiles = my_items * nk;            // key tiles this CTA streams

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      const bool all = i == B_SF0 || i == B_SF1 || i == B_P0 || i == B_P1 || i == B_OF0 || i == B_OF1 ||
                       i == B_OW0 || i == B_OW1;
      const bool both_issuers = i == B_QE0 || i == B_QE1 || i == B_KE0 || i == B_KE1 || i == B_VE0 || i == B_VE1;
      mbar_init(BAR(i), all ? 128 : both_issuers ? 2 : 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *holder;
  // set-up done: the next kernel may start its own; then wait for the inputs
  pdl_trigger();
  pdl_wait();

  // item li of this CTA -> (row*H + head, first query tile, query tiles in the item: 1 or 2)
  auto item_of = [&](int li, int& rh, int& qt0, int& ng) {
    const int it = static_cast<int>(blockIdx.x) + li * static_cast<int>(gridDim.x);
    rh = it / pairs;
    qt0 = (it - rh * pairs) * 2;
    ng = qt0 + 1 < nq ? 2 : 1;
  };

  if (warp < 4) {
    regs_dec<C::REG_CTRL>();
    if (warp == 0 && lane == 0) {  // ---------- loads: Q per item; K_n and V_n^T through two-stage rings
      // One fixed order (Q of an item, then K_n, V_n of each of its key tiles) with blocking
      // bounded waits, so the thread sleeps instead of polling next to the softmax warps.
      // Each wait depends only on MMAs whose operands were loaded earlier in this order.
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int n = 0;  // key tile of this CTA
      bool ok = true;
      for (int li = 0; li < my_items && ok; ++li) {
        int rh, qt0, ng;
        item_of(li, rh, qt0, ng);
        // Q of item li into buffer li & 1 once every Q K^T of item li-2 (its last user) completed;
        // issued after the previous item's K / V tiles, so it arrives while that item computes
        const int qbuf = li & 1, quse = li >> 1;
        if (quse > 0 && !mbar_wait(BAR(B_QE0 + qbuf), (quse - 1) & 1, status)) break;
        mbar_arrive_expect_tx(BAR(B_QF0 + qbuf), ng * C::QK_TILE);
        for (int g = 0; g < ng; ++g) {
          const int row0 = rh * a.Tpad + (qt0 + g) * 128;
          const uint32_t dst = sbase + C::OFF_Q + qbuf * C::Q_BUF + g * C::QK_TILE;
          tma_load_2d(dst, &tmQ, BAR(B_QF0 + qbuf), 0, row0);
          if (C::TAIL) tma_load_2d(dst + C::MAIN, &tmQt, BAR(B_QF0 + qbuf), 64, row0);
        }
        for (int j = 0; j < nk; ++j, ++n) {
          const uint32_t st = n & 1, free_parity = ((n >> 1) & 1) ^ 1u;
          // stage n & 1 is free once the MMA that read tile n-2 from it completed
          if (n >= 2 && !mbar_wait(BAR(B_KE0 + st), free_parity, status)) {
            ok = false;
            break;
          }
          const uint32_t kdst = sbase + C::OFF_K + st * C::QK_TILE;
          mbar_arrive_expect_tx(BAR(B_KF0 + st), C::QK_TILE);
          tma_load_2d(kdst, &tmK, BAR(B_KF0 + st), 0, rh * a.Tpad + j * 128);
          if (C::TAIL) tma_load_2d(kdst + C::MAIN, &tmKt, BAR(B_KF0 + st), 64, rh * a.Tpad + j * 128);
          if (n >= 2 && !mbar_wait(BAR(B_VE0 + st), free_parity, status)) {
            ok = false;
            break;
          }
          const uint32_t vdst = sbase + C::OFF_V + st * C::V_TILE;
          mbar_arrive_expect_tx(BAR(B_VF0 + st), C::V_TILE);
          tma_load_2d(vdst, &tmV, BAR(B_VF0 + st), j * 128, rh * C::DP);
          tma_load_2d(vdst + C::V_ATOM, &tmV, BAR(B_VF0 + st), j * 128 + 64, rh * C::DP);
        }
      }
    } else if ((warp == 1 || warp == 2) && lane == 0) {  // ---- MMA issuers: warp 1 group 0, warp 2 group 1
      // One issuing thread per query group, so neither group's MMAs queue behind the other's
      // and each issuer's serial chain stays short.  The shared K / V stages and the Q buffer
      // are released by both issuers (barrier count 2); an issuer whose group has no part in
      // an item still releases them (a commit with nothing new to track), and every release
      // comes after the matching full-barrier wait, so no issuer can run two phases ahead.
      const int g = warp - 1;
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, C::DP);
      // No division in the per-tile path: items and key tiles are followed by cursors, and
      // every descriptor is a constant high word plus base + offset.
      const uint32_t qb0 = sdesc_lo(sbase + C::OFF_Q) + g * (C::QK_TILE >> 4);
      const uint32_t k_lo = sdesc_lo(sbase + C::OFF_K), v_lo = sdesc_lo(sbase + C::OFF_V);
      const uint32_t pb = sdesc_lo(sbase + C::OFF_P) + g * (C::P_TILE >> 4);
      const uint32_t tS = tmem_base + g * 128, tO = tmem_base + 256 + g * 128;
      const int pmod = static_cast<int>(gridDim.x) % pairs;
      struct Cursor {
        int li, j, pidx, ng;  // item, key tile in the item, query-tile pair of the item, groups
      };
      auto first = [&]() {
        Cursor c{0, 0, static_cast<int>(blockIdx.x) % pairs, 0};
        c.ng = 2 * c.pidx + 1 < nq ? 2 : 1;
        return c;
      };
      auto advance = [&](Cursor& c) {
        if (++c.j == nk) {
          c.j = 0;
          ++c.li;
          c.pidx += pmod;
          if (c.pidx >= pairs) c.pidx -= pairs;
          c.ng = 2 * c.pidx + 1 < nq ? 2 : 1;
        }
      };
      int qk_cnt = 0, pv_cnt = 0, it_cnt = 0;  // this group's Q K^T, P V and started items
      Cursor cq = first(), cp = first();
      // S_g = Q_g K_n^T (cursor cq is at tile n)
      auto issue_qk = [&](int n) -> bool {
        const int qbuf = cq.li & 1;
        if (cq.j == 0 && !mbar_wait(BAR(B_QF0 + qbuf), (cq.li >> 1) & 1, status)) return false;
        if (!mbar_wait(BAR(B_KF0 + (n & 1)), (n >> 1) & 1, status)) return false;
        const uint32_t qb = qb0 + qbuf * (C::Q_BUF >> 4);
        if (g < cq.ng) {
          // S_g may be overwritten once the softmax of group g has read its previous tile
          if (qk_cnt > 0 && !mbar_wait(BAR(B_SF0 + g), (qk_cnt - 1) & 1, status)) return false;
          tc_fence_after();
          const uint32_t kb = k_lo + (n & 1) * (C::QK_TILE >> 4);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_ss(tS, sdesc_make(qb + 2 * k, kSdescHiSw128), sdesc_make(kb + 2 * k, kSdescHiSw128), idesc_s,
                        k > 0 ? 1u : 0u);
          if (C::TAIL)
            mma_bf16_ss(tS, sdesc_make(qb + (C::MAIN >> 4), kSdescHiSw32), sdesc_make(kb + (C::MAIN >> 4), kSdescHiSw32),
                        idesc_s, 1u);
          mma_commit(BAR(B_S0 + g));
          ++qk_cnt;
        }
        mma_commit(BAR(B_KE0 + (n & 1)));
        if (cq.j == nk - 1) mma_commit(BAR(B_QE0 + qbuf));
        advance(cq);
        return true;
      };
      // O_g (+)= P_g V_n (cursor cp is at tile n)
      auto issue_pv = [&](int n) -> bool {
        if (!mbar_wait(BAR(B_VF0 + (n & 1)), (n >> 1) & 1, status)) return false;
        if (g < cp.ng) {
          const bool first_tile = cp.j == 0;
          if (!mbar_wait(BAR(B_P0 + g), pv_cnt & 1, status)) return false;
          // a new item overwrites O_g: its epilogue for the previous item must have read it
          if (first_tile && it_cnt > 0 && !mbar_wait(BAR(B_OF0 + g), (it_cnt - 1) & 1, status)) return false;
          tc_fence_after();
          const uint32_t vb = v_lo + (n & 1) * (C::V_TILE >> 4);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_bf16_ss(tO, sdesc_make(pb + (k >> 2) * (C::MAIN >> 4) + (k & 3) * 2, kSdescHiSw128),
                        sdesc_make(vb + (k >> 2) * (C::V_ATOM >> 4) + (k & 3) * 2, kSdescHiSw128), idesc_o,
                        (!first_tile || k > 0) ? 1u : 0u);
          mma_commit(BAR(B_O0 + g));
          ++pv_cnt;
          if (first_tile) ++it_cnt;
        }
        mma_commit(BAR(B_VE0 + (n & 1)));
        advance(cp);
        return true;
      };
      // Q K^T of the next key tile goes in before P V of the current one, so the tensor
      // cores work while the softmax runs, across item boundaries too: the next item's Q sits
      // in the other Q buffer, loaded after this item's K / V tiles, and its first K / V
      // stage is freed by earlier MMAs only, so that Q K^T never waits on this P V.
      int n_qk = 0;
      bool ok = true;
      // Group 1 starts about half a key-tile period behind group 0 (once group 0 has written
      // its first P), so that the two groups' exp2 phases alternate on the MUFU pipe instead
      // of coinciding; group 0 needs nothing from group 1 to get there.
      if (g == 1 && !mbar_wait(BAR(B_GO), 0, status)) ok = false;
      for (int n = 0; n < ntiles && ok; ++n) {
        while (ok && (n_qk <= n || (n_qk == n + 1 && n_qk < ntiles))) ok = issue_qk(n_qk++);
        if (ok) ok = issue_pv(n);
      }
    }
  } else {  // ------------------------------- softmax / output: group g = warps 4-7 / 8-11
    regs_inc<C::REG_SOFTMAX>();
    const int g = (warp - 4) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;  // query row within the tile
    const uint32_t tS = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + g * 128;
    const uint32_t tO = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + 256 + g * 128;
    const float sc = 1.4426950408889634f * rsqrtf(static_cast<float>(DH));
    const uint32_t prow = sbase + C::OFF_P + g * C::P_TILE + r * 128;
    const uint32_t r7 = static_cast<uint32_t>(r & 7);
    const uint32_t ostage = sbase + C::OFF_P + g * C::P_TILE;  // the group's P buffer, between items
    const bool issuer = q == 0 && lane == 0;  // issues this group's output stores
    int cnt = 0;  // tiles of this group processed
    int ne = 0;   // items of this group finished
    bool ok = true;
    for (int li = 0; li < my_items && ok; ++li) {
      int rh, qt0, ng;
      item_of(li, rh, qt0, ng);
      if (g >= ng) continue;
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < nk; ++j, ++cnt) {
        ok = mbar_wait(BAR(B_S0 + g), cnt & 1, status);
        __syncwarp();
        if (__any_sync(0xffffffffu, !ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, s + c * 32);
        tmem_ld_wait<128>(s);
        tc_fence_before();
        mbar_arrive(BAR(B_SF0 + g));  // S_g is in registers: the next Q K^T may overwrite it

        // row maximum with eight independent partial maxima
        const int kvalid = a.T - j * 128;
        if (kvalid < 128) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= kvalid) s[i] = __float_as_uint(-INFINITY);
        }
        float mp[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) mp[e] = fmaxf(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1]));
#pragma unroll
        for (int i = 8; i < 128; i += 8)
#pragma unroll
          for (int e = 0; e < 4; ++e) mp[e] = max3f(mp[e], __uint_as_float(s[i + 2 * e]), __uint_as_float(s[i + 2 * e + 1]));
        const float mx = fmaxf(max3f(mp[0], mp[1], mp[2]), mp[3]);
        const float m_new = fmaxf(m_ref, mx * sc);
        // lazy rescale: the reference maximum moves (and O with it) only when the row maximum
        // grew by more than 2^8
        bool rescale = false;
        float alpha = 1.f;
        if (j == 0) {
          m_ref = m_new;
        } else if (__any_sync(0xffffffffu, m_new - m_ref > 8.0f)) {
          rescale = true;
          alpha = ex2_approx(m_ref - m_new);
          m_ref = m_new;
          if (lane == 0 && status != nullptr) atomicAdd(status + 1, 1);  // diagnostic event count
        }
        // P = 2^(s*sc - m_ref) as packed bf16 in registers (paired f32 scaling and row sums)
        uint32_t pk[64];
        const uint64_t sc2 = f2_pack(sc, sc), nm2 = f2_pack(-m_ref, -m_ref);
        uint64_t rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])), sc2, nm2);
          uint64_t p2;
          if (i % kEx2PolyEvery == kEx2PolyEvery - 1) {  // this pair on the FMA pipe (MUFU relief)
            p2 = ex2_poly_f2(x2);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
          }
          rs2[i & 1] = f2_add(rs2[i & 1], p2);
          float p0, p1;
          f2_unpack(p2, p0, p1);
          pk[i] = pack_bf16x2(p0, p1);
        }
        // the previous P V must be complete before O is rescaled and the P buffer rewritten;
        // at an item's first key tile the P buffer also held the previous item's output
        // staging tile, which its TMA store must have finished reading
        if (cnt > 0) {
          bool okw = mbar_wait(BAR(B_O0 + g), (cnt - 1) & 1, status);
          if (j == 0 && ne > 0) okw = okw && mbar_wait(BAR(B_OS0 + g), (ne - 1) & 1, status);
          __syncwarp();
          if (__any_sync(0xffffffffu, !okw)) {
            ok = false;
            break;
          }
        }
        if (rescale) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < C::DP / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(tO + c * 16, o);
            tmem_ld_wait<16>(o);
            const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
            for (int i = 0; i < 16; i += 2)
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2),
                        reinterpret_cast<float&>(o[i]), reinterpret_cast<float&>(o[i + 1]));
            tmem_st16(tO + c * 16, o);
          }
          tmem_st_wait();
          l *= alpha;
        }
        float r0, r1, r2, r3;
        f2_unpack(rs2[0], r0, r1);
        f2_unpack(rs2[1], r2, r3);
        l += (r0 + r1) + (r2 + r3);
        // P into the 128B-swizzled K-major layout the P V MMA reads
#pragma unroll
        for (int ch = 0; ch < 16; ++ch)
          st_shared_v4(prow + (ch >> 3) * C::MAIN + (((ch & 7) ^ r7) << 4), pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2],
                       pk[4 * ch + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(B_P0 + g));
        if (g == 0 && cnt == 0 && q == 0 && lane == 0) mbar_arrive(BAR(B_GO));
      }
      if (!ok) break;
      // item epilogue: O_g / l through shared memory to global memory (one TMA store)
      const bool okw = mbar_wait(BAR(B_O0 + g), (cnt - 1) & 1, status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !okw)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t o[C::DP];
#pragma unroll
      for (int c = 0; c < C::DP / 16; ++c) tmem_ld16(tO + c * 16, *reinterpret_cast<uint32_t(*)[16]>(o + c * 16));
      tmem_ld_wait<C::DP>(o);
      tc_fence_before();
      mbar_arrive(BAR(B_OF0 + g));  // O_g is in registers: the next item may overwrite it
      // the last P V has read the P buffer: it becomes this item's output staging tile
      const float inv = 1.0f / l;
      const uint32_t orow = ostage + r * C::O_ROW;
#pragma unroll
      for (int c = 0; c < DH / 8; ++c) {
        const uint32_t off = C::O_SW128 ? ((static_cast<uint32_t>(c) ^ r7) << 4) : static_cast<uint32_t>(c) * 16u;
        st_shared_v4(orow + off,
                     pack_bf16x2(__uint_as_float(o[c * 8 + 0]) * inv, __uint_as_float(o[c * 8 + 1]) * inv),
                     pack_bf16x2(__uint_as_float(o[c * 8 + 2]) * inv, __uint_as_float(o[c * 8 + 3]) * inv),
                     pack_bf16x2(__uint_as_float(o[c * 8 + 4]) * inv, __uint_as_float(o[c * 8 + 5]) * inv),
                     pack_bf16x2(__uint_as_float(o[c * 8 + 6]) * inv, __uint_as_float(o[c * 8 + 7]) * inv));
      }
      fence_proxy_async_smem();
      mbar_arrive(BAR(B_OW0 + g));
      if (issuer) {
        if (!mbar_wait(BAR(B_OW0 + g), ne & 1, status)) {
          ok = false;
        } else {
          const int row = rh / a.H, head = rh - row * a.H;
          tma_store_3d(&tmO, ostage, head * DH, (qt0 + g) * 128, row);  // rows past T are clipped
          bulk_commit_group();
          bulk_wait_read_all();         // the staging tile has been read: P may be written again
          mbar_arrive(BAR(B_OS0 + g));
        }
      }
      ++ne;
    }
    if (issuer) bulk_wait_all();
  }
  __syncwarp();  // lane-divergent roles reconverge before the block barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
#undef BAR
}

bool make_attention_maps(AttnMaps* m, const void* q, const void* k, const void* v, void* o, int R, int H, int T,
                         int Tpad, int dh, int DP, int d) {
  const uint64_t qrows = static_cast<uint64_t>(R) * H * Tpad;
  bool ok = make_tmap_bf16(&m->q, q, qrows, DP, 64, 128, 128) && make_tmap_bf16(&m->k, k, qrows, DP, 64, 128, 128) &&
            make_tmap_bf16(&m->v, v, static_cast<uint64_t>(R) * H * DP, Tpad, 64, DP, 128) &&
            make_tmap_bf16_3d(&m->o, o, d, T, R, dh, 128, dh * 2 == 128 ? 128 : 0);
  if (DP > 64)
    ok = ok && make_tmap_bf16(&m->qt, q, qrows, DP, 16, 128, 32) && make_tmap_bf16(&m->kt, k, qrows, DP, 16, 128, 32);
  else {
    m->qt = m->q;
    m->kt = m->k;
  }
  return ok;
}

template <int DH>
static cudaError_t launch_dh(const AttnArgs& a, const AttnMaps& mp, int* status, cudaStream_t st) {
  using C = AttnCfg<DH>;
  // one-time set-up per device: the shared-memory attribute is a per-device setting
  static int sms_of[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (sms_of[dev] == 0) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    // the register split (setmaxnreg) must fit in the launch allocation, or it would wait forever
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, attn_tc_kernel<DH>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * C::THREADS < C::REG_POOL) return cudaErrorInvalidConfiguration;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return cudaErrorInvalidDevice;
    sms_of[dev] = n;
  }
  const int num_sms = sms_of[dev];
  const int nq = a.Tpad / 128;
  const int items = a.R * a.H * ((nq + 1) / 2);
  const int grid = items < num_sms ? items : num_sms;
  if (grid == 0) return cudaSuccess;
  return launch_kernel(attn_tc_kernel<DH>, dim3(grid), dim3(C::THREADS), C::SMEM, st, mp.q, mp.qt, mp.k, mp.kt, mp.v,
                       mp.o, a, status);
}

cudaError_t launch_attention_tc(const AttnArgs& a, const AttnMaps& maps, int* status, cudaStream_t st) {
  if (a.Tpad % 128 != 0 || a.DP != (a.dh + 15) / 16 * 16) return cudaErrorInvalidValue;
  if (a.dh == 72) return launch_dh<72>(a, maps, status, st);
  if (a.dh == 64) return launch_dh<64>(a, maps, status, st);
  return cudaErrorInvalidValue;
}

}  // namespace dit
