// CUDA-core kernels of the DiT forward: condition MLP, patch embedding, fused
// LayerNorm + modulate, the float32 GEMM / attention of the fp32 path, the decoder
// fused with unpatchify and classifier-free guidance, and set-up tables.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dit {

bool g_pdl = true;

// ============================================================================ condition
// E[r, i]: timestep sinusoid [cos(t' f_i) | sin(t' f_i)], f_i = 10000^(-i/half),
// t' = t[b] * t_scale, in double so the argument (up to ~1000 rad) keeps full accuracy.
__global__ void cond_sinusoid_kernel(const float* __restrict__ t, int B, int R, int freq, float t_scale,
                                     float* __restrict__ E) {
  pdl_trigger();
  pdl_wait();
  const int half = freq / 2;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < R * freq; idx += gridDim.x * blockDim.x) {
    const int r = idx / freq, i = idx - r * freq;
    const int b = r % B;
    const int k = i < half ? i : i - half;
    const double f = exp(-log(10000.0) * static_cast<double>(k) / static_cast<double>(half));
    const double arg = static_cast<double>(t[b]) * static_cast<double>(t_scale) * f;
    E[idx] = static_cast<float>(i < half ? cos(arg) : sin(arg));
  }
}

// out[r, j] = act(sum_i W[j, i] in[r, i] + b[j]) (+ e(y_r) for the condition's second
// layer).  One warp per (output feature j, group of kRowsPerWarp rows): lanes split the
// K-long dot products, so the weight row is read once per row group.
constexpr int kRowsPerWarp = 8;

__device__ __forceinline__ void rows_dot(const float* __restrict__ w, const float* __restrict__ in, int K, int r0,
                                         int nr, int lane, float (&acc)[kRowsPerWarp]) {
#pragma unroll
  for (int q = 0; q < kRowsPerWarp; ++q) acc[q] = 0.f;
  for (int i = lane; i < K; i += 32) {
    const float wi = __ldg(w + i);
#pragma unroll
    for (int q = 0; q < kRowsPerWarp; ++q)
      if (q < nr) acc[q] = fmaf(wi, in[static_cast<size_t>(r0 + q) * K + i], acc[q]);
  }
#pragma unroll
  for (int q = 0; q < kRowsPerWarp; ++q) acc[q] = warp_sum(acc[q]);
}

template <bool SILU>
__global__ void rows_linear_kernel(const float* __restrict__ in, const float* __restrict__ W,
                                   const float* __restrict__ b, float* __restrict__ out, int R, int K, int N) {
  pdl_trigger();
  pdl_wait();
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int groups = (R + kRowsPerWarp - 1) / kRowsPerWarp;
  if (gw >= N * groups) return;
  const int j = gw / groups, r0 = (gw - j * groups) * kRowsPerWarp;
  const int nr = min(kRowsPerWarp, R - r0);
  float acc[kRowsPerWarp];
  rows_dot(W + static_cast<size_t>(j) * K, in, K, r0, nr, lane, acc);
  if (lane == 0) {
#pragma unroll
    for (int q = 0; q < kRowsPerWarp; ++q)
      if (q < nr) {
        const float v = acc[q] + b[j];
        out[static_cast<size_t>(r0 + q) * N + j] = SILU ? silu_f(v) : v;
      }
  }
}

// c[r, j] = W2 hid[r] + b2 + e(y_r);  sc = SiLU(c) (bf16 or f32).
// Rows r >= B of a guided batch take the null label num_classes.
__global__ void cond_out_kernel(CondArgs a) {
  pdl_trigger();
  pdl_wait();
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int groups = (a.R + kRowsPerWarp - 1) / kRowsPerWarp;
  if (gw >= a.d * groups) return;
  const int j = gw / groups, r0 = (gw - j * groups) * kRowsPerWarp;
  const int nr = min(kRowsPerWarp, a.R - r0);
  float acc[kRowsPerWarp];
  rows_dot(a.w2 + static_cast<size_t>(j) * a.d, a.hid, a.d, r0, nr, lane, acc);
  if (lane == 0) {
#pragma unroll
    for (int q = 0; q < kRowsPerWarp; ++q) {
      if (q >= nr) continue;
      const int r = r0 + q;
      float v = acc[q] + a.b2[j];
      if (a.cond_kind == DIT_COND_CLASS) {
        int lab;
        if (r < a.B) {
          lab = static_cast<const int*>(a.y)[r];
          if (lab < 0 || lab > a.num_classes) {
            record_status(a.status, DIT_ERR_BAD_LABEL);
            lab = lab < 0 ? 0 : a.num_classes;
          }
        } else {
          lab = a.num_classes;
        }
        v += a.table[static_cast<size_t>(lab) * a.d + j];
      } else {
        v += static_cast<const float*>(a.y)[static_cast<size_t>(r % a.B) * a.d + j];
      }
      if (a.c) a.c[static_cast<size_t>(r) * a.d + j] = v;
      const float sv = silu_f(v);
      if (a.sc_bf16)
        static_cast<uint16_t*>(a.sc)[static_cast<size_t>(r) * a.d + j] = f32_to_bf16(sv);
      else
        static_cast<float*>(a.sc)[static_cast<size_t>(r) * a.d + j] = sv;
    }
  }
}

cudaError_t launch_condition(const CondArgs& a, cudaStream_t st) {
  const int n = a.R * a.freq;
  cudaError_t e = launch_kernel(cond_sinusoid_kernel, dim3((n + 255) / 256), dim3(256), 0, st, a.t, a.B, a.R, a.freq,
                                 a.t_scale, a.E);
  if (e != cudaSuccess) return e;
  const int groups = (a.R + kRowsPerWarp - 1) / kRowsPerWarp;
  const int warps = a.d * groups;
  e = launch_kernel(rows_linear_kernel<true>, dim3((warps + 7) / 8), dim3(256), 0, st, (const float*)a.E, a.w1, a.b1,
                    a.hid, a.R, a.freq, a.d);
  if (e != cudaSuccess) return e;
  return launch_kernel(cond_out_kernel, dim3((warps + 7) / 8), dim3(256), 0, st, a);
}

// ============================================================================ patch embed
// h[(r*T + tau), j] = sum_k W[j, k] patch_k(r, tau) + b[j] (+ pos[tau, j]).
// Block: 16 tokens of one row; patch vectors gathered to shared memory first.
constexpr int kPatchTok = 16;
__global__ void patch_embed_kernel(PatchArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float sp[];  // [kPatchTok][Kp]
  const int gh = a.H / a.ph, gw = a.W / a.pw, gf = a.F / a.pt;
  const int T = gf * gh * gw;
  const int Kp = a.C * a.pt * a.ph * a.pw;
  const int r = blockIdx.y;
  const int b = r % a.B;
  const int tau0 = blockIdx.x * kPatchTok;
  const int ntok = min(kPatchTok, T - tau0);
  for (int idx = threadIdx.x; idx < ntok * Kp; idx += blockDim.x) {
    const int tl = idx / Kp, k = idx - tl * Kp;
    const int tau = tau0 + tl;
    const int f = tau / (gh * gw), i = (tau / gw) % gh, jj = tau % gw;
    const int iw = k % a.pw, ih = (k / a.pw) % a.ph, it = (k / (a.pw * a.ph)) % a.pt, c = k / (a.pw * a.ph * a.pt);
    const size_t xi = ((((static_cast<size_t>(b) * a.C + c) * a.F + f * a.pt + it) * a.H + i * a.ph + ih) * a.W) +
                      jj * a.pw + iw;
    sp[tl * Kp + k] = a.x[xi];
  }
  __syncthreads();
  for (int j = threadIdx.x; j < a.d; j += blockDim.x) {
    float acc[kPatchTok];
#pragma unroll
    for (int t = 0; t < kPatchTok; ++t) acc[t] = 0.f;
    const float* w = a.w + static_cast<size_t>(j) * Kp;
    for (int k = 0; k < Kp; ++k) {
      const float wk = __ldg(w + k);
#pragma unroll
      for (int t = 0; t < kPatchTok; ++t) acc[t] = fmaf(wk, sp[t * Kp + k], acc[t]);
    }
    const float bj = a.b[j];
    for (int t = 0; t < ntok; ++t) {
      float v = acc[t] + bj;
      if (a.pos) v += a.pos[static_cast<size_t>(tau0 + t) * a.d + j];
      a.h[(static_cast<size_t>(r) * T + tau0 + t) * a.d + j] = v;
    }
  }
}

cudaError_t launch_patch_embed(const PatchArgs& a, cudaStream_t st) {
  const int T = (a.F / a.pt) * (a.H / a.ph) * (a.W / a.pw);
  const int Kp = a.C * a.pt * a.ph * a.pw;
  const size_t smem = static_cast<size_t>(kPatchTok) * Kp * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(patch_embed_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid((T + kPatchTok - 1) / kPatchTok, a.R);
  return launch_kernel(patch_embed_kernel, grid, dim3(256), smem, st, a);
}

// ============================================================================ LN + modulate
// u = (h - mean) / sqrt(var + 1e-6) * (1 + scale[r]) + shift[r]  (population variance).
// One warp per token row, four rows per 128-thread block: the row's float4 loads are
// all issued before any use, mean and variance are two exact passes over registers,
// and u leaves as 8-byte (bf16) or 16-byte (f32) stores.  The pass is bound by the
// memory system: 6 bytes per element for the bf16 output.
constexpr int kLnMaxVec = 12;  // d <= 1536 (float4 per lane)
constexpr int kLnRowsPerBlock = 4;

template <bool BF16OUT>
__global__ void __launch_bounds__(32 * kLnRowsPerBlock) ln_modulate_kernel(LnArgs a) {
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x * kLnRowsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= a.M) return;
  const int nv = a.d >> 2;
  const float4* hp = reinterpret_cast<const float4*>(a.h + static_cast<size_t>(m) * a.d);
  float4 x[kLnMaxVec];
#pragma unroll
  for (int k = 0; k < kLnMaxVec; ++k) {
    const int c = lane + 32 * k;
    x[k] = c < nv ? hp[c] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < kLnMaxVec; ++k) sum += (x[k].x + x[k].y) + (x[k].z + x[k].w);
  const float mean = warp_sum(sum) / a.d;
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < kLnMaxVec; ++k) {
    const int c = lane + 32 * k;
    if (c < nv) {
      const float dx = x[k].x - mean, dy = x[k].y - mean, dz = x[k].z - mean, dw = x[k].w - mean;
      q += (dx * dx + dy * dy) + (dz * dz + dw * dw);
    }
  }
  const float rstd = rsqrtf(warp_sum(q) / a.d + 1e-6f);
  const int r = m / a.T;
  const float4* sh = reinterpret_cast<const float4*>(a.shift + static_cast<size_t>(r) * a.ld_mod);
  const float4* sc = reinterpret_cast<const float4*>(a.scale + static_cast<size_t>(r) * a.ld_mod);
#pragma unroll
  for (int k = 0; k < kLnMaxVec; ++k) {
    const int c = lane + 32 * k;
    if (c < nv) {
      const float4 s4 = __ldg(sc + c), b4 = __ldg(sh + c);
      float4 o;
      o.x = (x[k].x - mean) * rstd * (1.f + s4.x) + b4.x;
      o.y = (x[k].y - mean) * rstd * (1.f + s4.y) + b4.y;
      o.z = (x[k].z - mean) * rstd * (1.f + s4.z) + b4.z;
      o.w = (x[k].w - mean) * rstd * (1.f + s4.w) + b4.w;
      if (BF16OUT) {
        uint2 p;
        p.x = pack_bf16x2(o.x, o.y);
        p.y = pack_bf16x2(o.z, o.w);
        reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.u) + static_cast<size_t>(m) * a.d)[c] = p;
      } else {
        reinterpret_cast<float4*>(static_cast<float*>(a.u) + static_cast<size_t>(m) * a.d)[c] = o;
      }
    }
  }
}

cudaError_t launch_ln_modulate(const LnArgs& a, cudaStream_t st) {
  if ((a.d & 3) != 0 || a.d > 4 * 32 * kLnMaxVec) return cudaErrorInvalidValue;
  const int grid = (a.M + kLnRowsPerBlock - 1) / kLnRowsPerBlock;
  if (grid == 0) return cudaSuccess;
  if (a.u_bf16)
    return launch_kernel(ln_modulate_kernel<true>, dim3(grid), dim3(32 * kLnRowsPerBlock), 0, st, a);
  return launch_kernel(ln_modulate_kernel<false>, dim3(grid), dim3(32 * kLnRowsPerBlock), 0, st, a);
}

// ============================================================================ f32 GEMM
// D[M, N] = A[M, K] B[N, K]^T + epilogue; 64x64 tiles, 16-deep K slices, 4x4 per thread.
__device__ __forceinline__ void simt_epilogue(int epi, const EpiArgs& ea, int m, int n, float acc) {
  if (m >= ea.M || n >= ea.N) return;
  switch (epi) {
    case EPI_F32:
      static_cast<float*>(ea.out)[static_cast<size_t>(m) * ea.ldo + n] = acc + (ea.bias ? ea.bias[n] : 0.f);
      break;
    case EPI_ADALN:
      static_cast<float*>(ea.out)[static_cast<size_t>(n) * ea.ldo + m] = acc + ea.bias[m];
      break;
    case EPI_GELU:
      static_cast<float*>(ea.out)[static_cast<size_t>(m) * ea.ldo + n] = gelu_tanh_accurate(acc + ea.bias[n]);
      break;
    case EPI_RESID: {
      const int row = m / ea.T;
      const float g = ea.gate[static_cast<size_t>(row) * ea.ld_gate + n];
      float* hp = ea.h + static_cast<size_t>(m) * ea.ldh + n;
      *hp = fmaf(g, acc + ea.bias[n], *hp);
      break;
    }
    case EPI_QKV: {
      const int which = n / ea.d;
      const int head = (n - which * ea.d) / ea.dh;
      const int j = n - which * ea.d - head * ea.dh;
      const int row = m / ea.T, tok = m - row * ea.T;
      float* base = static_cast<float*>(which == 0 ? ea.q : (which == 1 ? ea.k : ea.v));
      base[(static_cast<size_t>(row * ea.H + head) * ea.T + tok) * ea.dh + j] = acc + ea.bias[n];
      break;
    }
    default:
      break;
  }
}

__global__ void __launch_bounds__(256) gemm_simt_kernel(int epi, const float* __restrict__ A,
                                                        const float* __restrict__ B, int K, EpiArgs ea) {
  pdl_trigger();
  pdl_wait();
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int idx = threadIdx.x; idx < 64 * 16; idx += 256) {
      const int rr = idx >> 4, kk = idx & 15;
      const int gm = m0 + rr, gn = n0 + rr, gk = k0 + kk;
      As[kk][rr] = (gm < ea.M && gk < K) ? A[static_cast<size_t>(gm) * K + gk] : 0.f;
      Bs[kk][rr] = (gn < ea.N && gk < K) ? B[static_cast<size_t>(gn) * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[kk][ty * 4 + i];
        bv[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) simt_epilogue(epi, ea, m0 + ty * 4 + i, n0 + tx * 4 + j, acc[i][j]);
}

cudaError_t launch_gemm_simt(int epi, const float* A, const float* B, int M, int N, int K, const EpiArgs& ea,
                             cudaStream_t st) {
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  return launch_kernel(gemm_simt_kernel, grid, dim3(256), 0, st, epi, A, B, K, ea);
}

// ============================================================================ f32 QK-norm + RoPE
__global__ void qknorm_rope_kernel(QkNormArgs a) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);  // one warp per (which, rh, tok)
  const int lane = threadIdx.x & 31;
  const int total = 2 * a.RH * a.T;
  if (row >= total) return;
  const int which = row / (a.RH * a.T);
  const int rem = row - which * a.RH * a.T;
  const int tok = rem % a.T;
  float* x = (which == 0 ? a.q : a.k) + static_cast<size_t>(rem) * a.dh;
  const float* g = which == 0 ? a.qn : a.kn;
  if (g) {
    float ss = 0.f;
    for (int j = lane; j < a.dh; j += 32) ss += x[j] * x[j];
    const float rs = rsqrtf(warp_sum(ss) / a.dh + 1e-6f);
    __syncwarp();
    for (int j = lane; j < a.dh; j += 32) x[j] = x[j] * rs * g[j];
    __syncwarp();
  }
  if (a.rope) {
    const float* rp = a.rope + static_cast<size_t>(tok) * a.dh;
    for (int i = lane; i < a.dh / 2; i += 32) {
      const float c = rp[2 * i], s = rp[2 * i + 1];
      const float x0 = x[2 * i], x1 = x[2 * i + 1];
      x[2 * i] = x0 * c - x1 * s;
      x[2 * i + 1] = x0 * s + x1 * c;
    }
  }
}

cudaError_t launch_qknorm_rope_f32(const QkNormArgs& a, cudaStream_t st) {
  const int rows = 2 * a.RH * a.T;
  return launch_kernel(qknorm_rope_kernel, dim3((rows + 7) / 8), dim3(256), 0, st, a);
}

// ============================================================================ SIMT attention
// One thread per query, 128 queries per block, keys/values staged 32 at a time in
// shared memory; online softmax in base 2 with the 1/sqrt(dh) scale folded into q.
template <int DH, bool BF16>
__global__ void __launch_bounds__(128) attn_simt_kernel(AttnArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float Ks[32][DH];
  __shared__ float Vs[32][DH];
  const int rh = blockIdx.y;
  const int row = rh / a.H, head = rh - row * a.H;
  const int qi = blockIdx.x * 128 + threadIdx.x;
  const int qrows = BF16 ? a.Tpad : a.T;
  const int ldq = BF16 ? a.DP : DH;
  const float qscale = rsqrtf(static_cast<float>(DH)) * 1.4426950408889634f;
  float q[DH], acc[DH];
  float mrun = -INFINITY, lrun = 0.f;
#pragma unroll
  for (int j = 0; j < DH; ++j) acc[j] = 0.f;
  if (qi < a.T) {
    const size_t off = (static_cast<size_t>(rh) * qrows + qi) * ldq;
#pragma unroll
    for (int j = 0; j < DH; ++j)
      q[j] = (BF16 ? bf16_to_f32(static_cast<const uint16_t*>(a.q)[off + j]) : static_cast<const float*>(a.q)[off + j]) *
             qscale;
  } else {
#pragma unroll
    for (int j = 0; j < DH; ++j) q[j] = 0.f;
  }
  for (int kt = 0; kt < a.T; kt += 32) {
    for (int idx = threadIdx.x; idx < 32 * DH; idx += 128) {
      const int kk = idx / DH, j = idx - kk * DH;
      const int key = kt + kk;
      float kv = 0.f, vv = 0.f;
      if (key < a.T) {
        if (BF16) {
          kv = bf16_to_f32(static_cast<const uint16_t*>(a.k)[(static_cast<size_t>(rh) * a.Tpad + key) * a.DP + j]);
          vv = bf16_to_f32(static_cast<const uint16_t*>(a.v)[(static_cast<size_t>(rh) * a.DP + j) * a.Tpad + key]);
        } else {
          kv = static_cast<const float*>(a.k)[(static_cast<size_t>(rh) * a.T + key) * DH + j];
          vv = static_cast<const float*>(a.v)[(static_cast<size_t>(rh) * a.T + key) * DH + j];
        }
      }
      Ks[kk][j] = kv;
      Vs[kk][j] = vv;
    }
    __syncthreads();
    float s[32];
    float mx = mrun;
#pragma unroll
    for (int kk = 0; kk < 32; ++kk) {
      float dot = 0.f;
#pragma unroll
      for (int j = 0; j < DH; ++j) dot = fmaf(q[j], Ks[kk][j], dot);
      s[kk] = (kt + kk < a.T) ? dot : -INFINITY;
      mx = fmaxf(mx, s[kk]);
    }
    const float corr = exp2f(mrun - mx);
    lrun *= corr;
#pragma unroll
    for (int j = 0; j < DH; ++j) acc[j] *= corr;
#pragma unroll
    for (int kk = 0; kk < 32; ++kk) {
      const float p = exp2f(s[kk] - mx);
      lrun += p;
#pragma unroll
      for (int j = 0; j < DH; ++j) acc[j] = fmaf(p, Vs[kk][j], acc[j]);
    }
    mrun = mx;
    __syncthreads();
  }
  if (qi < a.T) {
    const float inv = 1.f / lrun;
    const size_t off = (static_cast<size_t>(row) * a.T + qi) * a.d + static_cast<size_t>(head) * DH;
    if (BF16) {
      uint16_t* o = static_cast<uint16_t*>(a.o) + off;
#pragma unroll
      for (int j = 0; j < DH; ++j) o[j] = f32_to_bf16(acc[j] * inv);
    } else {
      float* o = static_cast<float*>(a.o) + off;
#pragma unroll
      for (int j = 0; j < DH; ++j) o[j] = acc[j] * inv;
    }
  }
}

cudaError_t launch_attention_simt(const AttnArgs& a, cudaStream_t st) {
  dim3 grid((a.T + 127) / 128, a.R * a.H);
  if (a.dh == 64) {
    return a.bf16 ? launch_kernel(attn_simt_kernel<64, true>, grid, dim3(128), 0, st, a)
                  : launch_kernel(attn_simt_kernel<64, false>, grid, dim3(128), 0, st, a);
  } else if (a.dh == 72) {
    return a.bf16 ? launch_kernel(attn_simt_kernel<72, true>, grid, dim3(128), 0, st, a)
                  : launch_kernel(attn_simt_kernel<72, false>, grid, dim3(128), 0, st, a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ============================================================================ decoder + unpatchify + CFG
// One block per (sample b, token tau).  Each warp computes decoder outputs p
// (stride 8); lanes split the d-long dot products.  Guided: both rows b and b+B
// are decoded and combined as z_null + s (z_cond - z_null) (on channels c < gch only
// when gch > 0; the others keep z_cond) before the scatter to
// out[b, c, f*pt+it, i*ph+ih, j*pw+iw] with p = ((it*ph + ih)*pw + iw)*Cout + c.
__global__ void decode_cfg_kernel(DecodeArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float su[];  // [2][d]
  const int tau = blockIdx.x, b = blockIdx.y;
  const int rows = a.guided ? 2 : 1;
  for (int idx = threadIdx.x; idx < rows * a.d; idx += blockDim.x) {
    const int rr = idx / a.d, j = idx - rr * a.d;
    const size_t m = static_cast<size_t>(b + rr * a.B) * a.T + tau;
    su[idx] = a.u_bf16 ? bf16_to_f32(static_cast<const uint16_t*>(a.u)[m * a.d + j])
                       : static_cast<const float*>(a.u)[m * a.d + j];
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int gw = a.W / a.pw, gh = a.H / a.ph;
  const int f = tau / (gh * gw), gi = (tau / gw) % gh, gj = tau % gw;
  for (int p = warp; p < a.P; p += nw) {
    const float* w = a.w + static_cast<size_t>(p) * a.d;
    float zc = 0.f, zu = 0.f;
    for (int j = lane; j < a.d; j += 32) {
      const float wj = __ldg(w + j);
      zc = fmaf(wj, su[j], zc);
      if (a.guided) zu = fmaf(wj, su[a.d + j], zu);
    }
    zc = warp_sum(zc);
    zu = warp_sum(zu);
    if (lane == 0) {
      const int c = p % a.Cout;
      zc += a.b[p];
      float val = zc;
      if (a.guided && (a.gch <= 0 || c < a.gch)) {
        zu += a.b[p];
        val = zu + a.s * (zc - zu);
      }
      const int iw = (p / a.Cout) % a.pw, ih = (p / (a.Cout * a.pw)) % a.ph, it = p / (a.Cout * a.pw * a.ph);
      const size_t oi = ((((static_cast<size_t>(b) * a.Cout + c) * a.F + f * a.pt + it) * a.H + gi * a.ph + ih) * a.W) +
                        gj * a.pw + iw;
      a.out[oi] = val;
    }
  }
}

cudaError_t launch_decode_cfg(const DecodeArgs& a, cudaStream_t st) {
  dim3 grid(a.T, a.B);
  const size_t smem = 2 * static_cast<size_t>(a.d) * sizeof(float);
  return launch_kernel(decode_cfg_kernel, grid, dim3(256), smem, st, a);
}

// ============================================================================ sampler step
// x_next = c0 x + c1 pred over [B, n_sample]; pred rows are ld_pred apart (the first C
// channels of a C_out-channel denoiser output).  Grid-stride, 16-byte accesses when every
// row start is 16-byte aligned.  x_next may alias x: each element is read, then written,
// by the same thread.
template <bool VEC>
__global__ void __launch_bounds__(256) sampler_step_kernel(SamplerArgs a) {
  pdl_trigger();
  pdl_wait();
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  if (VEC) {
    const long long per = a.n_sample >> 2, ld = a.ld_pred >> 2, total = per * a.B;
    const float4* x = reinterpret_cast<const float4*>(a.x);
    const float4* p = reinterpret_cast<const float4*>(a.pred);
    float4* o = reinterpret_cast<float4*>(a.x_next);
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
      const long long b = i / per, r = i - b * per;
      const float4 xv = x[i], pv = p[b * ld + r];
      o[i] = make_float4(fmaf(a.c0, xv.x, a.c1 * pv.x), fmaf(a.c0, xv.y, a.c1 * pv.y), fmaf(a.c0, xv.z, a.c1 * pv.z),
                         fmaf(a.c0, xv.w, a.c1 * pv.w));
    }
  } else {
    const long long total = a.n_sample * a.B;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
      const long long b = i / a.n_sample, r = i - b * a.n_sample;
      a.x_next[i] = fmaf(a.c0, a.x[i], a.c1 * a.pred[b * a.ld_pred + r]);
    }
  }
}

cudaError_t launch_sampler_step(const SamplerArgs& a, int num_sms, cudaStream_t st) {
  if (a.B <= 0 || a.n_sample <= 0) return cudaSuccess;
  const bool vec = (a.n_sample % 4) == 0 && (a.ld_pred % 4) == 0 && (reinterpret_cast<uintptr_t>(a.x) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(a.pred) & 15u) == 0 && (reinterpret_cast<uintptr_t>(a.x_next) & 15u) == 0;
  const long long work = vec ? a.n_sample / 4 * a.B : a.n_sample * a.B;
  const long long want = (work + 255) / 256;
  const int grid = static_cast<int>(want < 4LL * num_sms ? want : 4LL * num_sms);
  if (vec) return launch_kernel(sampler_step_kernel<true>, dim3(grid), dim3(256), 0, st, a);
  return launch_kernel(sampler_step_kernel<false>, dim3(grid), dim3(256), 0, st, a);
}

// ============================================================================ set-up tables
// pos[tau, :] (2D sin-cos, images): first d/2 dims encode the grid row, the last d/2
// the column; each half [sin(p w_k) | cos(p w_k)], w_k = 10000^(-k/(d/4)).
// rope[tau, i, :] = (cos, sin) of the angle of pair i: slice a = 2i / (dh/3) picks the
// axis (frame, row, col), k = (2i mod dh/3) / 2, angle = coord_a * 10000^(-2k/(dh/3)).
__global__ void pos_tables_kernel(float* pos, float* rope, int gf, int gh, int gw, int d, int dh) {
  const int T = gf * gh * gw;
  const int q = d / 4;
  if (pos) {
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < T * d; idx += gridDim.x * blockDim.x) {
      const int tau = idx / d, j = idx - tau * d;
      const int half = j / (d / 2), jj = j - half * (d / 2);
      const int p = half == 0 ? (tau / gw) % gh : tau % gw;
      const int k = jj % q;
      const double w = pow(10000.0, -static_cast<double>(k) / q);
      pos[idx] = static_cast<float>(jj < q ? sin(p * w) : cos(p * w));
    }
  }
  if (rope) {
    const int sl = dh / 3;
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < T * (dh / 2); idx += gridDim.x * blockDim.x) {
      const int tau = idx / (dh / 2), i = idx - tau * (dh / 2);
      const int axis = (2 * i) / sl, k = ((2 * i) % sl) / 2;
      const int coord = axis == 0 ? tau / (gh * gw) : (axis == 1 ? (tau / gw) % gh : tau % gw);
      const double ang = coord * pow(10000.0, -2.0 * k / sl);
      rope[2 * idx] = static_cast<float>(cos(ang));
      rope[2 * idx + 1] = static_cast<float>(sin(ang));
    }
  }
}

cudaError_t launch_pos_tables(float* pos, float* rope, int gf, int gh, int gw, int d, int dh, cudaStream_t st) {
  pos_tables_kernel<<<256, 256, 0, st>>>(pos, rope, gf, gh, gw, d, dh);
  return cudaGetLastError();
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ src, uint16_t* __restrict__ dst, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[i] = f32_to_bf16(src[i]);
}

cudaError_t launch_f32_to_bf16(const float* src, uint16_t* dst, size_t n, cudaStream_t st) {
  f32_to_bf16_kernel<<<1184, 256, 0, st>>>(src, dst, n);
  return cudaGetLastError();
}

// Waits on *flag (never set by anyone) with a bounded spin; records a timeout.
__global__ void wait_probe_kernel(int* flag, int* status, long long limit_ns) {
  if (threadIdx.x != 0) return;
  const uint64_t t0 = global_timer_ns();
  while (atomicAdd(flag, 0) == 0) {
    if (global_timer_ns() - t0 > static_cast<uint64_t>(limit_ns)) {
      record_status(status, DIT_ERR_DEVICE_TIMEOUT);
      return;
    }
    __nanosleep(1000);
  }
}

cudaError_t launch_wait_probe(int* flag, int* status, long long limit_ns, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(flag, status, limit_ns);
  return cudaGetLastError();
}

}  // namespace dit
