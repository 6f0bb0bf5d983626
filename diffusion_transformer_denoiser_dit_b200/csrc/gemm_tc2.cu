// Tensor-core GEMM on SM pairs (tcgen05 cta_group::2): D[M, N] = A[M, K] B[N, K]^T
// with 256 x BN output tiles, bf16 operands, float32 accumulation in tensor memory
// and the DiT epilogues fused in.
//
// A cluster of two CTAs runs on the two SMs of a TPC.  Per 64-wide K stage each CTA
// TMA-loads its own 128 rows of A and its own BN/2 rows of B (no multicast); both
// loads signal the leader CTA's "full" barrier.  One thread of the leader issues
// tcgen05.mma.cta_group::2 (M = 256, N = BN, K = 16): the tensor cores of both SMs
// work on the tile, each reading its own A rows and both halves of B, and each SM's
// TMEM receives its 128 rows of the accumulator.  The MMA completion is committed to
// the "empty" barrier of both CTAs (the stage may be refilled) and, at the end of a
// tile, to the "tmem full" barrier of both CTAs (their epilogues may read), one commit
// per CTA.  Each CTA's eight epilogue warps release the accumulator by arriving on the
// leader's "tmem empty" barrier.  Per SM and stage this moves 16 KB of A and BN*64 bytes of B
// for 128 x BN x 64 multiply-adds, half the B traffic of a one-SM tile.
// Persistent: one cluster per SM pair, tiles strided over clusters, two TMEM
// accumulators so the epilogue of one tile overlaps the main loop of the next.
// Every wait is bounded.
#include "common.cuh"
#include "gemm_epilogue.cuh"
#include "internal.h"

namespace dit {

template <int BN, int EPI>
struct Tc2Cfg {
  static constexpr int BK = 64;
  static constexpr int A_BYTES = 128 * BK * 2;         // this CTA's 128 rows of A
  static constexpr int B_BYTES = (BN / 2) * BK * 2;    // this CTA's BN/2 rows of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGING = epi_staged<EPI>() ? kEpilogueWarps * kStageBytesPerWarp : 0;
  static constexpr int BAR_BYTES = 256;
  static constexpr int STAGES_FIT = (232448 - 1024 - BAR_BYTES - STAGING) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int ACC_COLS = 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int SMEM = STAGES * STAGE_BYTES + STAGING + BAR_BYTES + 1024;
  static_assert(BN % 32 == 0 || BN == 144, "the pair splits B in two halves of whole 8-row groups");
  static_assert((BN / 2) % 8 == 0 && BN <= 256 && BN >= 32, "tile width");
  static_assert(B_BYTES % 1024 == 0, "stage tiles must stay 1024-byte aligned");
  static_assert(SMEM <= 232448, "dynamic shared memory above the sm_100 limit");
};

template <int BN, int EPI>
__global__ void __launch_bounds__(320, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const int K, const EpiArgs ea) {
  using C = Tc2Cfg<BN, EPI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + C::STAGING);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 4);
  const uint32_t bar0 = smem_u32(bars);
#define FULL_BAR(s) (bar0 + 8u * (s))
#define EMPTY_BAR(s) (bar0 + 8u * (C::STAGES + (s)))
#define TFULL_BAR(a) (bar0 + 8u * (2 * C::STAGES + (a)))
#define TEMPTY_BAR(a) (bar0 + 8u * (2 * C::STAGES + 2 + (a)))

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int m_tiles = (ea.M + 255) / 256;
  const int n_tiles = (ea.N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int kblocks = (K + 63) / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(FULL_BAR(s), 1);
      mbar_init(EMPTY_BAR(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(TFULL_BAR(a), 1);
      mbar_init(TEMPTY_BAR(a), 512);  // 256 epilogue threads in each CTA of the pair
    }
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(holder), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *holder;
  // set-up done: the next kernel may start its own; then wait for the inputs
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {  // ---------------- TMA producer (both CTAs)
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += nclusters) {
        const int m0 = (tile % m_tiles) * 256 + 128 * static_cast<int>(rank);
        const int n0 = (tile / m_tiles) * BN + (BN / 2) * static_cast<int>(rank);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(EMPTY_BAR(s), ph ^ 1u, ea.status)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t full_leader = mapa_shared(FULL_BAR(s), 0);
          if (leader) mbar_arrive_expect_tx(FULL_BAR(s), 2 * C::STAGE_BYTES);
          tma_load_2d_pair(sa, &tmA, full_leader, kb * 64, m0);
          tma_load_2d_pair(sa + C::A_BYTES, &tmB, full_leader, kb * 64, n0);
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // stage tail: wait until every stage this CTA filled has been released, so no
      // commit from the leader is still on its way to this CTA's barriers
      for (int i = 0; i < C::STAGES && ok; ++i) {
        if (!mbar_wait(EMPTY_BAR(s), ph ^ 1u, ea.status)) break;
        if (++s == C::STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {  // ---------------- MMA issuer (leader CTA only)
      constexpr uint32_t idesc = idesc_bf16_f32(256, BN);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int it = 0;
      for (int tile = cid; tile < num_tiles && ok; tile += nclusters, ++it) {
        const int a = it & 1;
        const uint32_t uph = (it >> 1) & 1;
        if (!mbar_wait(TEMPTY_BAR(a), uph ^ 1u, ea.status)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + a * C::ACC_COLS;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(FULL_BAR(s), ph, ea.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_pair(dt, sdesc_k_sw128(sa + k * 32), sdesc_k_sw128(sb + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
          mma_commit_pair(EMPTY_BAR(s));
          mma_commit_pair(mapa_shared(EMPTY_BAR(s), 1));
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) {
          mma_commit_pair(TFULL_BAR(a));
          mma_commit_pair(mapa_shared(TFULL_BAR(a), 1));
        }
      }
      // accumulator tail: every epilogue release (including the partner CTA's remote
      // arrivals) has landed before this CTA may leave
      for (int i = (it >= 2 ? it - 2 : 0); i < it && ok; ++i)
        if (!mbar_wait(TEMPTY_BAR(i & 1), (i >> 1) & 1, ea.status)) break;
    }
  } else {  // ------------------------ epilogue warps 2..9 (both CTAs)
    const int q = warp & 3;
    int it = 0;
    for (int tile = cid; tile < num_tiles; tile += nclusters, ++it) {
      const int a = it & 1;
      const uint32_t uph = (it >> 1) & 1;
      const bool ok = mbar_wait(TFULL_BAR(a), uph, ea.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !ok)) break;
      tc_fence_after();
      const int m0 = (tile % m_tiles) * 256 + 128 * static_cast<int>(rank), n0 = (tile / m_tiles) * BN;
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * C::ACC_COLS;
      if constexpr (EPI == EPI_RESID_T)
        epilogue_resid_t<BN / 2>(ea, &tmC, tacc, m0 + q * 32, lane, n0, ((warp - 2) >> 2) * (BN / 2),
                                 staging + (warp - 2) * kStageBytesPerWarp);
      else if constexpr (EPI == EPI_QKV_T)
        epilogue_qkv_t<BN / 2>(ea, tacc, m0 + q * 32, lane, n0, ((warp - 2) >> 2) * (BN / 2),
                               staging + (warp - 2) * kStageBytesPerWarp);
      else if constexpr (epi_staged<EPI>())
        epilogue_cols_staged<BN / 2, EPI>(ea, tacc, m0 + q * 32, lane, n0, ((warp - 2) >> 2) * (BN / 2),
                                          staging + (warp - 2) * kStageBytesPerWarp);
      else
        epilogue_cols<BN / 2, (EPI == EPI_QKV_HEAD ? EPI_QKV : EPI), EPI == EPI_QKV_HEAD || EPI == EPI_XATTN>(
            ea, tacc, m0 + q * 32 + lane, n0, ((warp - 2) >> 2) * (BN / 2));
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(TEMPTY_BAR(a), 0));
    }
    if (epi_staged<EPI>() && lane == 0) bulk_wait_all();  // TMA stores of this warp are complete
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();  // no CTA leaves while its partner may still signal it or use its TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
#undef FULL_BAR
#undef EMPTY_BAR
#undef TFULL_BAR
#undef TEMPTY_BAR
}

template <int BN, int EPI>
static cudaError_t launch_pair_bn(const CUtensorMap* tA, const CUtensorMap* tB, const CUtensorMap* tC, int K,
                                  const EpiArgs& ea, int num_sms, cudaStream_t st) {
  using C = Tc2Cfg<BN, EPI>;
  static int clusters_of[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  int& max_clusters = clusters_of[dev];
  if (max_clusters == 0) {
    cudaError_t e =
        cudaFuncSetAttribute(gemm_tc2_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t qc = {};
    qc.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    qc.blockDim = dim3(320, 1, 1);
    qc.dynamicSmemBytes = C::SMEM;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    qc.attrs = qa;
    qc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel<BN, EPI>, &qc) != cudaSuccess || n <= 0) n = num_sms / 2;
    max_clusters = n;
  }
  const int tiles = ((ea.M + 255) / 256) * ((ea.N + BN - 1) / BN);
  if (tiles == 0) return cudaSuccess;
  const int clusters = tiles < max_clusters ? tiles : max_clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(320, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<BN, EPI>, *tA, *tB, tC ? *tC : *tB, K, ea);
}

int gemm_tc2_supported_bn(int bn) { return bn == 64 || bn == 128 || bn == 144 || bn == 192 || bn == 256; }

cudaError_t launch_gemm_tc2(int epi, int bn, const CUtensorMap* tA, const CUtensorMap* tB, int K, const EpiArgs& ea,
                            int num_sms, cudaStream_t st, const CUtensorMap* tC) {
  if (epi == EPI_RESID_T && tC == nullptr) return cudaErrorInvalidValue;
#define DIT_BN2_CASE(BNV, EPIV) \
  if (bn == BNV) return launch_pair_bn<BNV, EPIV>(tA, tB, tC, K, ea, num_sms, st);
  switch (epi) {
    case EPI_F32:
      DIT_BN2_CASE(64, EPI_F32) DIT_BN2_CASE(128, EPI_F32) DIT_BN2_CASE(144, EPI_F32) DIT_BN2_CASE(192, EPI_F32)
      DIT_BN2_CASE(256, EPI_F32) break;
    case EPI_GELU:
      DIT_BN2_CASE(128, EPI_GELU) DIT_BN2_CASE(256, EPI_GELU)
      break;
    case EPI_RESID_T:
      DIT_BN2_CASE(256, EPI_RESID_T) break;
    case EPI_QKV_T:
      DIT_BN2_CASE(256, EPI_QKV_T) break;
    default:
      break;
  }
#undef DIT_BN2_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dit
