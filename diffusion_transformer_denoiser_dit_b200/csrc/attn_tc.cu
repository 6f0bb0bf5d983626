// Tensor-core flash attention for sm_100a (full, non-causal, one head per CTA row).
//
// O = softmax(Q K^T / sqrt(dh)) V for a 128-query tile of one (sample row, head):
//   warp 0   one thread loads Q once, then K_j and V_j^T into two-stage rings (TMA,
//            no multicast); a stage is refilled as soon as the MMA that read it
//            completed (polled without blocking, so the K and V streams never wait on
//            each other).  For T <= 256 every tile is requested at the start.
//   warp 1   allocates 256 TMEM columns (S: 0..127, O: 128..) and one thread issues
//            S_j = Q K_j^T (M=128, N=128, K=dh padded to 80, both operands in shared
//            memory) and O += P_j V_j (M=128, N=DP, K=128) with P_j read from TMEM.
//   warps 2-5 one query row per thread: S_j from TMEM into registers, online softmax
//            in base 2 with lazy O rescaling (only when the running max grows by more
//            than 2^8), P_j as packed bf16 written back over the first 64 columns of
//            S (tcgen05.st), final O / l to global memory.
// Two CTAs fit on one SM (about 102 KB shared memory and 256 TMEM columns each), so
// one CTA's softmax overlaps the other's MMAs.
//
// Layouts: q, k [R*H, Tpad, DP] bf16 (rows of one head contiguous, head dim padded
// with zeros to DP = 80 for dh = 72); v transposed [R*H, DP, Tpad]; padded key rows
// are zero and masked to -inf in the last key tile.  o [R*T, d] bf16, token-major.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dit {

template <int DH>
struct AttnCfg {
  static constexpr int DP = (DH + 15) / 16 * 16;
  static constexpr bool TAIL = DP > 64;                 // head-dim columns 64..DP-1
  static constexpr int MAIN = 128 * 128;                // 128 rows x 64 bf16
  static constexpr int TAILB = TAIL ? 128 * 32 : 0;     // 128 rows x 16 bf16
  static constexpr int QK_TILE = MAIN + TAILB;          // one Q or K tile
  static constexpr int V_ATOM = DP * 128;               // DP rows x 64 keys
  static constexpr int V_TILE = 2 * V_ATOM;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QK_TILE;         // two K stages
  static constexpr int OFF_V = OFF_K + 2 * QK_TILE;     // two V^T stages
  static constexpr int OFF_BAR = OFF_V + 2 * V_TILE;
  static constexpr int SMEM = OFF_BAR + 128 + 1024;
  static constexpr int TMEM_COLS = 256;
  static constexpr int O_COL = 128;
  static_assert(QK_TILE % 1024 == 0 && V_ATOM % 1024 == 0, "1024-byte aligned tiles");
  static_assert(2 * (SMEM + 1024) <= 233472, "two CTAs per SM");
};

// barriers: Q loaded; K / V^T stage full and empty (two stages each); S ready; P ready; P V done
enum { B_Q = 0, B_KF0, B_KF1, B_KE0, B_KE1, B_VF0, B_VF1, B_VE0, B_VE1, B_S, B_P, B_O, B_COUNT };

template <int DH>
__global__ void __launch_bounds__(192, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQt,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKt,
                   const __grid_constant__ CUtensorMap tmV, const AttnArgs a, int* status) {
  using C = AttnCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  uint32_t* holder = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * B_COUNT);
#define BAR(i) (bar0 + 8u * (i))

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rh = blockIdx.y;
  const int qt = blockIdx.x;
  const int nk = (a.T + 127) / 128;

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) mbar_init(BAR(i), i == B_P ? 128 : 1);
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

  if (warp == 0) {
    if (lane == 0) {  // ---------------- loads: Q once; K_j and V_j^T into two-stage rings
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int qrow0 = rh * a.Tpad + qt * 128;
      const int vrow0 = rh * C::DP;
      mbar_arrive_expect_tx(BAR(B_Q), C::QK_TILE);
      tma_load_2d(sbase + C::OFF_Q, &tmQ, BAR(B_Q), 0, qrow0);
      if (C::TAIL) tma_load_2d(sbase + C::OFF_Q + C::MAIN, &tmQt, BAR(B_Q), 64, qrow0);
      int jk = 0, jv = 0;
      const uint64_t t0 = global_timer_ns();
      while (jk < nk || jv < nk) {
        // stage j&1 is free once the MMA that read its previous tile (j-2) completed
        if (jk < nk && (jk < 2 || mbar_test(BAR(B_KE0 + (jk & 1)), ((jk >> 1) & 1) ^ 1u))) {
          const uint32_t dst = sbase + C::OFF_K + (jk & 1) * C::QK_TILE;
          const int krow0 = rh * a.Tpad + jk * 128;
          mbar_arrive_expect_tx(BAR(B_KF0 + (jk & 1)), C::QK_TILE);
          tma_load_2d(dst, &tmK, BAR(B_KF0 + (jk & 1)), 0, krow0);
          if (C::TAIL) tma_load_2d(dst + C::MAIN, &tmKt, BAR(B_KF0 + (jk & 1)), 64, krow0);
          ++jk;
        }
        if (jv < nk && (jv < 2 || mbar_test(BAR(B_VE0 + (jv & 1)), ((jv >> 1) & 1) ^ 1u))) {
          const uint32_t dst = sbase + C::OFF_V + (jv & 1) * C::V_TILE;
          mbar_arrive_expect_tx(BAR(B_VF0 + (jv & 1)), C::V_TILE);
          tma_load_2d(dst, &tmV, BAR(B_VF0 + (jv & 1)), jv * 128, vrow0);
          tma_load_2d(dst + C::V_ATOM, &tmV, BAR(B_VF0 + (jv & 1)), jv * 128 + 64, vrow0);
          ++jv;
        }
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          record_status(status, DIT_ERR_DEVICE_TIMEOUT);
          break;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------- MMA issuer
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, C::DP);
      const uint32_t tS = tmem_base;
      const uint32_t tO = tmem_base + C::O_COL;
      bool ok = mbar_wait(BAR(B_Q), 0, status);
      for (int j = 0; j < nk && ok; ++j) {
        const int st = j & 1;
        const uint32_t use = (j >> 1) & 1;
        ok = mbar_wait(BAR(B_KF0 + st), use, status);
        // S (and P_{j-1}, which lives in S) may be overwritten once P_{j-1} V_{j-1} completed
        if (ok && j > 0) ok = mbar_wait(BAR(B_O), (j - 1) & 1, status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kb = sbase + C::OFF_K + st * C::QK_TILE;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16_ss(tS, sdesc_k_sw128(sbase + C::OFF_Q + k * 32), sdesc_k_sw128(kb + k * 32), idesc_s,
                      k > 0 ? 1u : 0u);
        if (C::TAIL) mma_bf16_ss(tS, sdesc_k_sw32(sbase + C::OFF_Q + C::MAIN), sdesc_k_sw32(kb + C::MAIN), idesc_s, 1u);
        mma_commit(BAR(B_S));
        mma_commit(BAR(B_KE0 + st));
        // O += P_j V_j: P_j (bf16, 64 TMEM columns over S) as the A operand
        ok = mbar_wait(BAR(B_P), j & 1, status) && mbar_wait(BAR(B_VF0 + st), use, status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t vb = sbase + C::OFF_V + st * C::V_TILE;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_bf16_ts(tO, tS + 8 * k, sdesc_k_sw128(vb + (k >> 2) * C::V_ATOM + (k & 3) * 32), idesc_o,
                      (j > 0 || k > 0) ? 1u : 0u);
        mma_commit(BAR(B_O));
        mma_commit(BAR(B_VE0 + st));
      }
    }
  } else {  // ------------------------------------------ softmax / output warps 2..5
    const int q = warp & 3;
    const int r = q * 32 + lane;  // query row within the tile
    const uint32_t tS = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t tO = tS + C::O_COL;
    const float sc = 1.4426950408889634f * rsqrtf(static_cast<float>(DH));
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      ok = mbar_wait(BAR(B_S), j & 1, status);
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
      const int kvalid = a.T - j * 128;
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        float v = __uint_as_float(s[i]);
        if (i >= kvalid) v = -INFINITY;
        s[i] = __float_as_uint(v);
        mx = fmaxf(mx, v);
      }
      const float m_new = fmaxf(m_ref, mx * sc);
      if (j == 0) {
        m_ref = m_new;
      } else if (__any_sync(0xffffffffu, m_new - m_ref > 8.0f)) {
        // lazy rescale: O only moves to the new reference when the maximum grew by more
        // than 2^8 (P_{j-1} V_{j-1} has completed: Q K_j^T was issued after it)
        const float alpha = ex2_approx(m_ref - m_new);
#pragma unroll
        for (int c = 0; c < C::DP / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tO + c * 16, o);
          tmem_ld_wait<16>(o);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st16(tO + c * 16, o);
        }
        l *= alpha;
        m_ref = m_new;
      }
      // P = 2^(s*sc - m_ref) as bf16 pairs, written over the first 64 columns of S
      float rs = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(s[half * 64 + 2 * e]), sc, -m_ref));
          const float p1 = ex2_approx(fmaf(__uint_as_float(s[half * 64 + 2 * e + 1]), sc, -m_ref));
          rs += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS + half * 32, pk);
      }
      tmem_st_wait();
      l += rs;
      tc_fence_before();
      mbar_arrive(BAR(B_P));
    }
    if (ok) {
      const bool okw = mbar_wait(BAR(B_O), (nk - 1) & 1, status);
      __syncwarp();
      if (!__any_sync(0xffffffffu, !okw)) {
        tc_fence_after();
        uint32_t o[C::DP];
#pragma unroll
        for (int c = 0; c < C::DP / 16; ++c) tmem_ld16(tO + c * 16, *reinterpret_cast<uint32_t(*)[16]>(o + c * 16));
        tmem_ld_wait<C::DP>(o);
        const int qi = qt * 128 + r;
        if (qi < a.T) {
          const float inv = 1.0f / l;
          const int row = rh / a.H, head = rh - row * a.H;
          uint16_t* dst = static_cast<uint16_t*>(a.o) + (static_cast<size_t>(row) * a.T + qi) * a.d + head * DH;
#pragma unroll
          for (int c = 0; c < DH / 8; ++c) {
            uint4 pk;
            pk.x = pack_bf16x2(__uint_as_float(o[c * 8 + 0]) * inv, __uint_as_float(o[c * 8 + 1]) * inv);
            pk.y = pack_bf16x2(__uint_as_float(o[c * 8 + 2]) * inv, __uint_as_float(o[c * 8 + 3]) * inv);
            pk.z = pack_bf16x2(__uint_as_float(o[c * 8 + 4]) * inv, __uint_as_float(o[c * 8 + 5]) * inv);
            pk.w = pack_bf16x2(__uint_as_float(o[c * 8 + 6]) * inv, __uint_as_float(o[c * 8 + 7]) * inv);
            *reinterpret_cast<uint4*>(dst + c * 8) = pk;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
#undef BAR
}

bool make_attention_maps(AttnMaps* m, const void* q, const void* k, const void* v, int RH, int Tpad, int DP) {
  const uint64_t qrows = static_cast<uint64_t>(RH) * Tpad;
  bool ok = make_tmap_bf16(&m->q, q, qrows, DP, 64, 128, 128) && make_tmap_bf16(&m->k, k, qrows, DP, 64, 128, 128) &&
            make_tmap_bf16(&m->v, v, static_cast<uint64_t>(RH) * DP, Tpad, 64, DP, 128);
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
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  dim3 grid(a.Tpad / 128, a.R * a.H);
  return launch_kernel(attn_tc_kernel<DH>, grid, dim3(192), C::SMEM, st, mp.q, mp.qt, mp.k, mp.kt, mp.v, a, status);
}

cudaError_t launch_attention_tc(const AttnArgs& a, const AttnMaps& maps, int* status, cudaStream_t st) {
  if (a.Tpad % 128 != 0 || a.DP != (a.dh + 15) / 16 * 16) return cudaErrorInvalidValue;
  if (a.dh == 72) return launch_dh<72>(a, maps, status, st);
  if (a.dh == 64) return launch_dh<64>(a, maps, status, st);
  return cudaErrorInvalidValue;
}

}  // namespace dit
