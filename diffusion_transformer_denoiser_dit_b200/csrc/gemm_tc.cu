// Tensor-core GEMM for sm_100a: D[M, N] = A[M, K] * B[N, K]^T, bf16 operands,
// float32 accumulation in tensor memory, with the DiT epilogues fused in.
//
// Design (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: 128x64 A tile + BNx64 B tile per stage, 128-byte
//               swizzle, STAGES-deep ring guarded by full/empty mbarriers.
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               (M=128, N=BN, K=16, four per 64-wide stage) into one of two TMEM
//               accumulators and commits stage releases / accumulator hand-off.
//   warps 2..5  epilogue: tcgen05.ld of its 32 TMEM lanes (one output row per
//               thread), bias / GELU / gated residual / head-major scatter with
//               QK-RMSNorm and 3D RoPE, stores to global memory.  Two accumulators
//               let the epilogue of tile i overlap the main loop of tile i+1.
// Every mbarrier wait is bounded (common.cuh); no TMA multicast is used.
#include "common.cuh"
#include "internal.h"

namespace dit {

template <int BN>
struct TcCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_FIT = (220 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int ACC_COLS = 256;  // TMEM column distance of the two accumulators
  static constexpr int TMEM_COLS = 512;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "tcgen05 M=128 needs N in [16, 256], N % 16 == 0");
  static_assert(B_BYTES % 1024 == 0, "stage tiles must stay 1024-byte aligned for the 128B swizzle");
  static_assert(SMEM <= 232448, "dynamic shared memory above the sm_100 limit");
};

// ------------------------------------------------------------------------- epilogues
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_tile(const EpiArgs& ea, uint32_t tacc, int m, int n0) {
  const bool mok = m < ea.M;
  if constexpr (EPI == EPI_QKV) {
    constexpr int DH = BN / 2;  // one tile = two whole heads of q, k or v
    static_assert(DH % 8 == 0, "head dim must be a multiple of 8");
#pragma unroll 1
    for (int g = 0; g < 2; ++g) {
      uint32_t r[DH];
#pragma unroll
      for (int c = 0; c < DH / 8; ++c) DIT_TMEM_LD_X8(tacc + g * DH + c * 8, (r + c * 8));
      tmem_ld_wait<DH>(r);
      const int n = n0 + g * DH;
      if (n >= ea.N) continue;
      const int which = n / ea.d;
      const int head = (n - which * ea.d) / DH;
      const int row = m / ea.T, tok = m - row * ea.T;
      float v[DH];
#pragma unroll
      for (int j = 0; j < DH; ++j) v[j] = __uint_as_float(r[j]) + __ldg(ea.bias + n + j);
      if (which < 2) {
        const float* gn = which == 0 ? ea.qn : ea.kn;
        if (gn != nullptr) {
          float ss = 0.f;
#pragma unroll
          for (int j = 0; j < DH; ++j) ss = fmaf(v[j], v[j], ss);
          const float rs = rsqrtf(ss * (1.0f / DH) + 1e-6f);
#pragma unroll
          for (int j = 0; j < DH; ++j) v[j] = v[j] * rs * __ldg(gn + j);
        }
        if (ea.rope != nullptr) {
          const float* rp = ea.rope + static_cast<size_t>(tok) * DH;
#pragma unroll
          for (int i = 0; i < DH / 2; ++i) {
            const float c = __ldg(rp + 2 * i), s = __ldg(rp + 2 * i + 1);
            const float x0 = v[2 * i], x1 = v[2 * i + 1];
            v[2 * i] = x0 * c - x1 * s;
            v[2 * i + 1] = x0 * s + x1 * c;
          }
        }
        if (mok) {
          uint16_t* dst = static_cast<uint16_t*>(which == 0 ? ea.q : ea.k) +
                          (static_cast<size_t>(row * ea.H + head) * ea.Tpad + tok) * ea.DP;
#pragma unroll
          for (int c = 0; c < DH / 8; ++c) {
            uint4 pk;
            pk.x = pack_bf16x2(v[c * 8 + 0], v[c * 8 + 1]);
            pk.y = pack_bf16x2(v[c * 8 + 2], v[c * 8 + 3]);
            pk.z = pack_bf16x2(v[c * 8 + 4], v[c * 8 + 5]);
            pk.w = pack_bf16x2(v[c * 8 + 6], v[c * 8 + 7]);
            *reinterpret_cast<uint4*>(dst + c * 8) = pk;
          }
        }
      } else if (mok) {
        uint16_t* dst = static_cast<uint16_t*>(ea.v) + static_cast<size_t>(row * ea.H + head) * ea.DP * ea.Tpad + tok;
#pragma unroll
        for (int j = 0; j < DH; ++j) dst[static_cast<size_t>(j) * ea.Tpad] = f32_to_bf16(v[j]);
      }
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < BN / 16; ++c) {
      uint32_t r[16];
      tmem_ld16(tacc + c * 16, r);
      tmem_ld_wait<16>(r);
      const int n = n0 + c * 16;
      if (!mok || n >= ea.N) continue;
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
      const bool full = (n + 16 <= ea.N);
      if constexpr (EPI == EPI_ADALN) {
        // rows of this GEMM are modulation features j = m, columns are sample rows
        const float bj = __ldg(ea.bias + m);
        float* o = static_cast<float*>(ea.out) + m;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (n + i < ea.N) o[static_cast<size_t>(n + i) * ea.ldo] = v[i] + bj;
      } else if constexpr (EPI == EPI_F32) {
        float* o = static_cast<float*>(ea.out) + static_cast<size_t>(m) * ea.ldo + n;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (n + i < ea.N) o[i] = v[i] + (ea.bias ? __ldg(ea.bias + n + i) : 0.f);
      } else if constexpr (EPI == EPI_GELU) {
        uint16_t* o = static_cast<uint16_t*>(ea.out) + static_cast<size_t>(m) * ea.ldo + n;
        if (full) {
          uint32_t p[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            p[i] = pack_bf16x2(gelu_tanh_fast(v[2 * i] + __ldg(ea.bias + n + 2 * i)),
                               gelu_tanh_fast(v[2 * i + 1] + __ldg(ea.bias + n + 2 * i + 1)));
          reinterpret_cast<uint4*>(o)[0] = make_uint4(p[0], p[1], p[2], p[3]);
          reinterpret_cast<uint4*>(o)[1] = make_uint4(p[4], p[5], p[6], p[7]);
        } else {
          for (int i = 0; i < 16 && n + i < ea.N; ++i) o[i] = f32_to_bf16(gelu_tanh_fast(v[i] + __ldg(ea.bias + n + i)));
        }
      } else if constexpr (EPI == EPI_RESID) {
        const int row = m / ea.T;
        const float* gt = ea.gate + static_cast<size_t>(row) * ea.ld_gate + n;
        float* hp = ea.h + static_cast<size_t>(m) * ea.ldh + n;
        if (full) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 g4 = __ldg(reinterpret_cast<const float4*>(gt) + i);
            const float4 b4 = __ldg(reinterpret_cast<const float4*>(ea.bias + n) + i);
            float4 h4 = reinterpret_cast<float4*>(hp)[i];
            h4.x = fmaf(g4.x, v[4 * i + 0] + b4.x, h4.x);
            h4.y = fmaf(g4.y, v[4 * i + 1] + b4.y, h4.y);
            h4.z = fmaf(g4.z, v[4 * i + 2] + b4.z, h4.z);
            h4.w = fmaf(g4.w, v[4 * i + 3] + b4.w, h4.w);
            reinterpret_cast<float4*>(hp)[i] = h4;
          }
        } else {
          for (int i = 0; i < 16 && n + i < ea.N; ++i) hp[i] = fmaf(gt[i], v[i] + ea.bias[n + i], hp[i]);
        }
      }
    }
  }
}

// ------------------------------------------------------------------------- kernel
template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const int K,
                   const EpiArgs ea) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 4);
  const uint32_t bar0 = smem_u32(bars);
  // barrier addresses: full[s], empty[s], tmem_full[a], tmem_empty[a]
#define FULL_BAR(s) (bar0 + 8u * (s))
#define EMPTY_BAR(s) (bar0 + 8u * (C::STAGES + (s)))
#define TFULL_BAR(a) (bar0 + 8u * (2 * C::STAGES + (a)))
#define TEMPTY_BAR(a) (bar0 + 8u * (2 * C::STAGES + 2 + (a)))

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (ea.M + 127) / 128;
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
      mbar_init(TEMPTY_BAR(a), 128);
    }
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

  if (warp == 0) {
    if (lane == 0) {  // ---------------- TMA producer
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % m_tiles) * 128, n0 = (tile / m_tiles) * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(EMPTY_BAR(s), ph ^ 1u, ea.status)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          mbar_arrive_expect_tx(FULL_BAR(s), C::STAGE_BYTES);
          tma_load_2d(sa, &tmA, FULL_BAR(s), kb * 64, m0);
          tma_load_2d(sa + C::A_BYTES, &tmB, FULL_BAR(s), kb * 64, n0);
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------- MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
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
            mma_bf16_ss(dt, sdesc_k_sw128(sa + k * 32), sdesc_k_sw128(sb + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
          mma_commit(EMPTY_BAR(s));
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) mma_commit(TFULL_BAR(a));
      }
    }
  } else {  // ------------------------ epilogue warps 2..5
    const int q = warp & 3;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int a = it & 1;
      const uint32_t uph = (it >> 1) & 1;
      const bool ok = mbar_wait(TFULL_BAR(a), uph, ea.status);
      __syncwarp();
      if (__any_sync(0xffffffffu, !ok)) break;
      tc_fence_after();
      const int m0 = (tile % m_tiles) * 128, n0 = (tile / m_tiles) * BN;
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * C::ACC_COLS;
      epilogue_tile<BN, EPI>(ea, tacc, m0 + q * 32 + lane, n0);
      tc_fence_before();
      mbar_arrive(TEMPTY_BAR(a));
    }
  }
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

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                    uint32_t box_rows, int swizzle_bytes) {
  PFN_encodeTiled_t fn = encode_fn();
  if (fn == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) != 0 || (cols * 2) % 16 != 0 || box_rows == 0 ||
      box_rows > 256 || box_cols == 0 || (box_cols * 2) % 16 != 0 || box_cols * 2 > (uint32_t)swizzle_bytes)
    return false;
  CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16_kmajor(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows) {
  return make_tmap_bf16(map, base, rows, K, 64, box_rows, 128);
}

template <int BN, int EPI>
static cudaError_t launch_bn(const CUtensorMap* tA, const CUtensorMap* tB, int K, const EpiArgs& ea, int num_sms,
                             cudaStream_t st) {
  using C = TcCfg<BN>;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const int tiles = ((ea.M + 127) / 128) * ((ea.N + BN - 1) / BN);
  if (tiles == 0) return cudaSuccess;
  const int grid = tiles < num_sms ? tiles : num_sms;
  gemm_tc_kernel<BN, EPI><<<grid, 192, C::SMEM, st>>>(*tA, *tB, K, ea);
  return cudaGetLastError();
}

int gemm_tc_supported_bn(int bn) {
  return bn == 16 || bn == 32 || bn == 64 || bn == 128 || bn == 144 || bn == 192 || bn == 256;
}

cudaError_t launch_gemm_tc(int epi, int bn, const CUtensorMap* tA, const CUtensorMap* tB, int K, const EpiArgs& ea,
                           int num_sms, cudaStream_t st) {
#define DIT_BN_CASE(BNV, EPIV) \
  if (bn == BNV) return launch_bn<BNV, EPIV>(tA, tB, K, ea, num_sms, st);
  switch (epi) {
    case EPI_F32:
      DIT_BN_CASE(16, EPI_F32) DIT_BN_CASE(32, EPI_F32) DIT_BN_CASE(64, EPI_F32) DIT_BN_CASE(128, EPI_F32)
      DIT_BN_CASE(144, EPI_F32) DIT_BN_CASE(192, EPI_F32) DIT_BN_CASE(256, EPI_F32) break;
    case EPI_ADALN:
      DIT_BN_CASE(16, EPI_ADALN) DIT_BN_CASE(32, EPI_ADALN) DIT_BN_CASE(64, EPI_ADALN)
      DIT_BN_CASE(128, EPI_ADALN) DIT_BN_CASE(256, EPI_ADALN) break;
    case EPI_GELU:
      DIT_BN_CASE(128, EPI_GELU) DIT_BN_CASE(144, EPI_GELU) DIT_BN_CASE(192, EPI_GELU) DIT_BN_CASE(256, EPI_GELU) break;
    case EPI_RESID:
      DIT_BN_CASE(128, EPI_RESID) DIT_BN_CASE(144, EPI_RESID) DIT_BN_CASE(192, EPI_RESID)
      DIT_BN_CASE(256, EPI_RESID) break;
    case EPI_QKV:
      DIT_BN_CASE(128, EPI_QKV) DIT_BN_CASE(144, EPI_QKV) break;
    default:
      break;
  }
#undef DIT_BN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dit
