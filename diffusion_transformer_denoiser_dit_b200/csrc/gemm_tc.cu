// Tensor-core GEMM for sm_100a: D[M, N] = A[M, K] * B[N, K]^T, bf16 operands,
// float32 accumulation in tensor memory, with the DiT epilogues fused in.
//
// Design (one persistent CTA per SM, 320 threads = 10 warps):
//   warp 0      TMA producer: 128 rows of A and BN rows of B per stage, 128 bytes of K
//               each (64 bf16 or 128 E4M3 elements), 128-byte swizzle, STAGES-deep ring
//               guarded by full/empty mbarriers.
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               (M=128, N=BN, K=16 bf16 or 32 E4M3, four per stage) into one of two TMEM
//               accumulators and commits stage releases / accumulator hand-off.
//   warps 2..9  epilogue: warp w reads TMEM lanes 32*(w%4)..+31 (one output row per
//               thread) and one half of the tile's columns (warps 2-5 the first half,
//               6-9 the second); bias / GELU / gated residual / head-major scatter with
//               QK-RMSNorm and 3D RoPE, stores to global memory.  Two accumulators let
//               the epilogue of tile i overlap the main loop of tile i+1.
// Every mbarrier wait is bounded (common.cuh); no TMA multicast is used.  When a wait
// runs out, the producer and the MMA issuer first wait (bounded again) for the copies
// and MMAs they already issued before the CTA frees its TMEM and exits.
#include "common.cuh"
#include "gemm_epilogue.cuh"
#include "internal.h"

namespace dit {

// k-blocks per split-K slice for a requested split (1 when not split); the slice count is then
// ceil(kblocks / result), so no slice is empty.
__host__ __device__ inline int kblocks_per_slice(int kblocks, int split) {
  return split > 1 && kblocks > 0 ? (kblocks + split - 1) / split : (kblocks > 0 ? kblocks : 1);
}

template <int BN, int EPI>
struct TcCfg {
  static constexpr bool F8 = epi_fp8<EPI>();            // E4M3 operands (one byte per element)
  static constexpr int BM = 128, BK = F8 ? 128 : 64;    // K elements per 128-byte stage row
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGING = epi_staged<EPI>() ? kEpilogueWarps * kStageBytesPerWarp : 0;
  static constexpr int BAR_BYTES = 256;
  static constexpr int STAGES_FIT = (232448 - 1024 - BAR_BYTES - STAGING) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int ACC_COLS = 256;  // TMEM column distance of the two accumulators
  static constexpr int TMEM_COLS = 512;
  static constexpr int SMEM = STAGES * STAGE_BYTES + STAGING + BAR_BYTES + 1024;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "tcgen05 M=128 needs N in [16, 256], N % 16 == 0");
  static_assert(B_BYTES % 1024 == 0, "stage tiles must stay 1024-byte aligned for the 128B swizzle");
  static_assert(SMEM <= 232448, "dynamic shared memory above the sm_100 limit");
  static_assert(STAGES >= 3, "pipeline too shallow");
};

// ------------------------------------------------------------------------- kernel
template <int BN, int EPI>
__global__ void __launch_bounds__(320, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const int K, const EpiArgs ea) {
  using C = TcCfg<BN, EPI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + C::STAGING);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 5);
  const uint32_t bar0 = smem_u32(bars);
  // barrier addresses: full[s], empty[s], tmem_full[a], tmem_empty[a]
#define FULL_BAR(s) (bar0 + 8u * (s))
#define EMPTY_BAR(s) (bar0 + 8u * (C::STAGES + (s)))
#define TFULL_BAR(a) (bar0 + 8u * (2 * C::STAGES + (a)))
#define TEMPTY_BAR(a) (bar0 + 8u * (2 * C::STAGES + 2 + (a)))
#define DRAIN_BAR (bar0 + 8u * (2 * C::STAGES + 4))

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (ea.M + 127) / 128;
  const int n_tiles = (ea.N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int kblocks_all = (K + C::BK - 1) / C::BK;
  // split-K (the reduce-add residual epilogues only): work unit u is k-slice u / num_tiles of
  // tile u % num_tiles, so the slices of one tile are far apart in time
  const int kblocks = kblocks_per_slice(kblocks_all, (EPI == EPI_RESID_T || EPI == EPI_RESID_T8) ? ea.ksplit : 1);
  const int num_units = num_tiles * ((kblocks_all + kblocks - 1) / kblocks);  // every slice has >= 1 k-block

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(FULL_BAR(s), 1);
      mbar_init(EMPTY_BAR(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(TFULL_BAR(a), 1);
      mbar_init(TEMPTY_BAR(a), 256);  // 8 epilogue warps
    }
    mbar_init(DRAIN_BAR, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
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
    if (lane == 0) {  // ---------------- TMA producer
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      uint32_t armed = 0;  // bit s: stage s has been filled at least once
      for (int unit = blockIdx.x; unit < num_units && ok; unit += gridDim.x) {
        const int tile = unit % num_tiles, kb0 = (unit / num_tiles) * kblocks;
        const int m0 = (tile % m_tiles) * 128, n0 = (tile / m_tiles) * BN;
        const int kb1 = min(kb0 + kblocks, kblocks_all);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(EMPTY_BAR(s), ph ^ 1u, ea.status)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          mbar_arrive_expect_tx(FULL_BAR(s), C::STAGE_BYTES);
          tma_load_2d(sa, &tmA, FULL_BAR(s), kb * C::BK, m0);
          tma_load_2d(sa + C::A_BYTES, &tmB, FULL_BAR(s), kb * C::BK, n0);
          armed |= 1u << s;
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        // a wait ran out: let every copy already issued land before shared memory is
        // released (the last fill of stage j used parity ph for j < s, ph ^ 1 for j >= s)
        for (int j = 0; j < C::STAGES; ++j)
          if (armed & (1u << j)) mbar_wait(FULL_BAR(j), j < s ? ph : ph ^ 1u, ea.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------- MMA issuer
      constexpr uint32_t idesc = C::F8 ? idesc_e4m3_f32(128, BN) : idesc_bf16_f32(128, BN);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int it = 0;
      for (int unit = blockIdx.x; unit < num_units && ok; unit += gridDim.x, ++it) {
        const int kb0 = (unit / num_tiles) * kblocks, nkb = min(kblocks, kblocks_all - kb0);
        const int a = it & 1;
        const uint32_t uph = (it >> 1) & 1;
        if (!mbar_wait(TEMPTY_BAR(a), uph ^ 1u, ea.status)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + a * C::ACC_COLS;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(FULL_BAR(s), ph, ea.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // four 32-byte K steps per 128-byte row
            if constexpr (C::F8)
              mma_e4m3_ss(dt, sdesc_k_sw128(sa + k * 32), sdesc_k_sw128(sb + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
            else
              mma_bf16_ss(dt, sdesc_k_sw128(sa + k * 32), sdesc_k_sw128(sb + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit(EMPTY_BAR(s));
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) mma_commit(TFULL_BAR(a));
      }
      if (!ok) {
        // a wait ran out: the MMAs already issued must finish before TMEM is freed
        mma_commit(DRAIN_BAR);
        mbar_wait(DRAIN_BAR, 0, ea.status);
      }
    }
  } else {  // ------------------------ epilogue warps 2..9
    const int q = warp & 3;
    int it = 0;
    for (int unit = blockIdx.x; unit < num_units; unit += gridDim.x, ++it) {
      const int tile = unit % num_tiles;
      const bool first_slice = unit < num_tiles;  // the bias is added once per tile
      const int a = it & 1;
      const uint32_t uph = (it >> 1) & 1;
      const bool ok = mbar_wait(TFULL_BAR(a), uph, ea.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !ok)) break;
      tc_fence_after();
      const int m0 = (tile % m_tiles) * 128, n0 = (tile / m_tiles) * BN;
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * C::ACC_COLS;
      if constexpr (EPI == EPI_RESID_T || EPI == EPI_RESID_T8)
        epilogue_resid_t<BN / 2, EPI == EPI_RESID_T8>(ea, &tmC, tacc, m0 + q * 32, lane, n0,
                                                       ((warp - 2) >> 2) * (BN / 2),
                                                       staging + (warp - 2) * kStageBytesPerWarp, first_slice);
      else if constexpr (EPI == EPI_GELU8)
        epilogue_gelu8<BN / 2>(ea, tacc, m0 + q * 32 + lane, n0, ((warp - 2) >> 2) * (BN / 2));
      else if constexpr (EPI == EPI_QKV_T || EPI == EPI_QKV_T8)
        epilogue_qkv_t<BN / 2, EPI == EPI_QKV_T8>(ea, tacc, m0 + q * 32, lane, n0, ((warp - 2) >> 2) * (BN / 2),
                               staging + (warp - 2) * kStageBytesPerWarp);
      else if constexpr (epi_staged<EPI>())
        epilogue_cols_staged<BN / 2, EPI>(ea, tacc, m0 + q * 32, lane, n0, ((warp - 2) >> 2) * (BN / 2),
                                          staging + (warp - 2) * kStageBytesPerWarp);
      else
        epilogue_cols<BN / 2, (EPI == EPI_QKV_HEAD ? EPI_QKV : EPI),
                      EPI == EPI_QKV_HEAD || EPI == EPI_QKV_HEAD8 || EPI == EPI_XATTN>(
            ea, tacc, m0 + q * 32 + lane, n0, ((warp - 2) >> 2) * (BN / 2));
      tc_fence_before();
      mbar_arrive(TEMPTY_BAR(a));
    }
    if (epi_staged<EPI>() && lane == 0) bulk_wait_all();  // TMA stores of this warp are complete
  }
  __syncwarp();  // lane-divergent roles reconverge before the block barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
#undef FULL_BAR
#undef EMPTY_BAR
#undef TFULL_BAR
#undef TEMPTY_BAR
#undef DRAIN_BAR
}

// ------------------------------------------------------------------------- host side
typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                      const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled_t encode_fn() {
  static PFN_encodeTiled_t fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled_t>(p);
  }
  return fn;
}

static bool make_tmap(CUtensorMap* map, CUtensorMapDataType dt, uint32_t esize, const void* base, uint64_t rows,
                      uint64_t cols, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes) {
  PFN_encodeTiled_t fn = encode_fn();
  if (fn == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) != 0 || (cols * esize) % 16 != 0 || box_rows == 0 ||
      box_rows > 256 || box_cols == 0 || (box_cols * esize) % 16 != 0 ||
      (swizzle_bytes > 0 && box_cols * esize > (uint32_t)swizzle_bytes))
    return false;
  CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                    uint32_t box_rows, int swizzle_bytes) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rows, cols, box_cols, box_rows, swizzle_bytes);
}

bool make_tmap_f32(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                   uint32_t box_rows, int swizzle_bytes) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, rows, cols, box_cols, box_rows, swizzle_bytes);
}

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0,
                       uint32_t box1, int swizzle_bytes) {
  PFN_encodeTiled_t fn = encode_fn();
  if (fn == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) != 0 || (d0 * 2) % 16 != 0 || box0 == 0 ||
      box0 > 256 || box1 == 0 || box1 > 256 || (box0 * 2) % 16 != 0 ||
      (swizzle_bytes > 0 && box0 * 2 > (uint32_t)swizzle_bytes))
    return false;
  CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16_kmajor(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows) {
  return make_tmap_bf16(map, base, rows, K, 64, box_rows, 128);
}

bool make_tmap_e4m3_kmajor(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, rows, K, 128, box_rows, 128);
}

template <int BN, int EPI>
static cudaError_t launch_bn(const CUtensorMap* tA, const CUtensorMap* tB, const CUtensorMap* tC, int K,
                             const EpiArgs& ea, int num_sms, cudaStream_t st) {
  using C = TcCfg<BN, EPI>;
  static bool attr_done[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int kb_all = (K + C::BK - 1) / C::BK;
  const int kb = kblocks_per_slice(kb_all, (EPI == EPI_RESID_T || EPI == EPI_RESID_T8) ? ea.ksplit : 1);
  const int tiles = ((ea.M + 127) / 128) * ((ea.N + BN - 1) / BN) * ((kb_all + kb - 1) / kb);
  if (tiles == 0) return cudaSuccess;
  const int grid = tiles < num_sms ? tiles : num_sms;
  return launch_kernel(gemm_tc_kernel<BN, EPI>, dim3(grid), dim3(320), C::SMEM, st, *tA, *tB, tC ? *tC : *tB, K, ea);
}

int gemm_tc_supported_bn(int bn) {
  return bn == 16 || bn == 32 || bn == 64 || bn == 128 || bn == 144 || bn == 192 || bn == 256;
}

cudaError_t launch_gemm_tc(int epi, int bn, const CUtensorMap* tA, const CUtensorMap* tB, int K, const EpiArgs& ea,
                           int num_sms, cudaStream_t st, const CUtensorMap* tC) {
  if ((epi == EPI_RESID_T || epi == EPI_RESID_T8) && tC == nullptr) return cudaErrorInvalidValue;
#define DIT_BN_CASE(BNV, EPIV) \
  if (bn == BNV) return launch_bn<BNV, EPIV>(tA, tB, tC, K, ea, num_sms, st);
  switch (epi) {
    case EPI_F32:
      DIT_BN_CASE(16, EPI_F32) DIT_BN_CASE(32, EPI_F32) DIT_BN_CASE(64, EPI_F32) DIT_BN_CASE(128, EPI_F32)
      DIT_BN_CASE(144, EPI_F32) DIT_BN_CASE(192, EPI_F32) DIT_BN_CASE(256, EPI_F32) break;
    case EPI_ADALN:
      DIT_BN_CASE(16, EPI_ADALN) DIT_BN_CASE(32, EPI_ADALN) DIT_BN_CASE(64, EPI_ADALN)
      DIT_BN_CASE(128, EPI_ADALN) DIT_BN_CASE(256, EPI_ADALN) break;
    case EPI_GELU:
      DIT_BN_CASE(128, EPI_GELU) DIT_BN_CASE(256, EPI_GELU) break;
    case EPI_QKV_HEAD:
      DIT_BN_CASE(128, EPI_QKV_HEAD) DIT_BN_CASE(144, EPI_QKV_HEAD) break;
    case EPI_RESID_T:
      DIT_BN_CASE(256, EPI_RESID_T) break;
    case EPI_QKV_T:
      DIT_BN_CASE(256, EPI_QKV_T) break;
    case EPI_XATTN:
      DIT_BN_CASE(128, EPI_XATTN) DIT_BN_CASE(144, EPI_XATTN) break;
    case EPI_F32_8:
      DIT_BN_CASE(64, EPI_F32_8) DIT_BN_CASE(128, EPI_F32_8) DIT_BN_CASE(256, EPI_F32_8) break;
    case EPI_GELU8:
      DIT_BN_CASE(256, EPI_GELU8) break;
    case EPI_RESID_T8:
      DIT_BN_CASE(256, EPI_RESID_T8) break;
    case EPI_QKV_T8:
      DIT_BN_CASE(256, EPI_QKV_T8) break;
    case EPI_QKV_HEAD8:
      DIT_BN_CASE(128, EPI_QKV_HEAD8) DIT_BN_CASE(144, EPI_QKV_HEAD8) break;
    default:
      break;
  }
#undef DIT_BN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dit
