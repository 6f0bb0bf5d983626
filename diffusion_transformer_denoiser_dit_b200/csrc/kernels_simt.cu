// CUDA-core kernels of the DiT forward: condition MLP, patch embedding, fused
// LayerNorm + modulate, the float32 GEMM / attention of the fp32 path, classifier-free
// guidance fused with unpatchify, and set-up tables.
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

// The condition MLP's two layers, out[r, j] = W[j] . in[r] + b[j] for all sample rows r.  A
// block of 8 warps owns 8 output features and a group of up to 32 rows.  The 8 weight rows are
// staged in shared memory once (coalesced float4 loads) and read back as broadcasts; warp w takes
// the w-th eighth of K for every row of the group (lane = row, its input row read as float4), so
// each 16-byte input load feeds 32 multiply-adds into 8 independent accumulators; the 8 partial
// sums of every (row, feature) are added through shared memory.  Thread t then owns row t / 8 and
// feature t % 8, so a warp's outputs are 4 rows of 8 consecutive features.
constexpr int kCondRows = 32, kCondFeat = 8, kCondWarps = 8;
constexpr int kCondRedLd = kCondFeat + 1;  // padded so the lanes' partial-sum writes hit distinct banks

// Dynamic shared memory of one block: the weight slab [kCondFeat][K] and the partial sums
// [kCondWarps][kCondRows][kCondRedLd].
__host__ __device__ inline size_t cond_smem_bytes(int K) {
  return (static_cast<size_t>(kCondFeat) * K + static_cast<size_t>(kCondWarps) * kCondRows * kCondRedLd) *
         sizeof(float);
}

// ws[f * K + k] = W[min(j0 + f, N - 1), k]  (K % 4 == 0; rows past N repeat the last one and are
// never stored)
__device__ __forceinline__ void cond_stage_w(const float* __restrict__ W, int N, int K, int j0, float* ws) {
  const int K4 = K >> 2;
  for (int i = threadIdx.x; i < kCondFeat * K4; i += blockDim.x) {
    const int f = i / K4, k4 = i - f * K4;
    const int j = min(j0 + f, N - 1);
    reinterpret_cast<float4*>(ws + f * K)[k4] = __ldg(reinterpret_cast<const float4*>(W + static_cast<size_t>(j) * K) + k4);
  }
}

// W[j0 + t % 8] . in[r0 + t / 8] for the calling thread t (0 when that row is past the group);
// every thread of the block calls it, and it leaves the partial-sum area free for the next call.
__device__ __forceinline__ float cond_dot8(const float* __restrict__ in, int K, int r0, int nr, const float* ws,
                                           float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K4 = K >> 2, per = (K4 + kCondWarps - 1) / kCondWarps;
  const int c0 = warp * per, c1 = min(c0 + per, K4);
  float acc[kCondFeat];
#pragma unroll
  for (int f = 0; f < kCondFeat; ++f) acc[f] = 0.f;
  if (lane < nr) {
    const float4* x = reinterpret_cast<const float4*>(in + static_cast<size_t>(r0 + lane) * K);
#pragma unroll 4
    for (int c = c0; c < c1; ++c) {
      const float4 v = x[c];
#pragma unroll
      for (int f = 0; f < kCondFeat; ++f) {
        const float4 w = reinterpret_cast<const float4*>(ws + f * K)[c];
        acc[f] = fmaf(v.w, w.w, fmaf(v.z, w.z, fmaf(v.y, w.y, fmaf(v.x, w.x, acc[f]))));
      }
    }
  }
  __syncthreads();  // the previous call's readers of red are done
#pragma unroll
  for (int f = 0; f < kCondFeat; ++f) red[(warp * kCondRows + lane) * kCondRedLd + f] = acc[f];
  __syncthreads();
  const int r = threadIdx.x / kCondFeat, f = threadIdx.x % kCondFeat;
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kCondWarps; ++w) s += red[(w * kCondRows + r) * kCondRedLd + f];
  return s;
}

// hid[r, j] = SiLU(W1[j] . E[r] + b1[j])
__global__ void __launch_bounds__(256) cond_hidden_kernel(const float* __restrict__ E, const float* __restrict__ W1,
                                                          const float* __restrict__ b1, float* __restrict__ hid, int R,
                                                          int K, int N) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float4 cond_smem4[];
  float* ws = reinterpret_cast<float*>(cond_smem4);
  float* red = ws + kCondFeat * K;
  const int j0 = blockIdx.x * kCondFeat;
  cond_stage_w(W1, N, K, j0, ws);
  __syncthreads();
  const int j = j0 + threadIdx.x % kCondFeat, rl = threadIdx.x / kCondFeat;
  for (int r0 = blockIdx.y * kCondRows; r0 < R; r0 += gridDim.y * kCondRows) {
    const int nr = min(kCondRows, R - r0);
    const float v = cond_dot8(E, K, r0, nr, ws, red);
    if (j < N && rl < nr) hid[static_cast<size_t>(r0 + rl) * N + j] = silu_f(v + b1[j]);
  }
}

// c[r, j] = e_t + e_y with e_t = W2[j] . hid[r] + b2[j] and e_y = e(y_r);  sc = SiLU(c) (bf16
// or f32); optionally e_t and e_y as condition tokens.  Rows r >= B of a guided batch take the
// null label num_classes.
__global__ void __launch_bounds__(256) cond_out_kernel(CondArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float4 cond_smem4[];
  float* ws = reinterpret_cast<float*>(cond_smem4);
  float* red = ws + kCondFeat * a.d;
  const int j0 = blockIdx.x * kCondFeat;
  cond_stage_w(a.w2, a.d, a.d, j0, ws);
  __syncthreads();
  const int j = j0 + threadIdx.x % kCondFeat, rl = threadIdx.x / kCondFeat;
  for (int r0 = blockIdx.y * kCondRows; r0 < a.R; r0 += gridDim.y * kCondRows) {
    const int nr = min(kCondRows, a.R - r0);
    const float acc = cond_dot8(a.hid, a.d, r0, nr, ws, red);
    if (j >= a.d || rl >= nr) continue;
    const int r = r0 + rl;
    const float et = acc + a.b2[j];  // timestep embedding
    float ey;                        // class embedding / text vector
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
      ey = a.table[static_cast<size_t>(lab) * a.d + j];
    } else {
      ey = static_cast<const float*>(a.y)[static_cast<size_t>(r % a.B) * a.d + j];
    }
    const float v = et + ey;
    if (a.c) a.c[static_cast<size_t>(r) * a.d + j] = v;
    if (a.sc) {
      const float sv = silu_f(v);
      if (a.sc_bf16)
        static_cast<uint16_t*>(a.sc)[static_cast<size_t>(r) * a.d + j] = f32_to_bf16(sv);
      else
        static_cast<float*>(a.sc)[static_cast<size_t>(r) * a.d + j] = sv;
    }
    if (a.tok_h) {
      a.tok_h[r * a.tok_ld + j] = et;
      a.tok_h[r * a.tok_ld + a.d + j] = ey;
    }
    if (a.ctx) {
      const size_t i0 = static_cast<size_t>(2 * r) * a.d + j, i1 = i0 + a.d;
      if (a.ctx_bf16) {
        static_cast<uint16_t*>(a.ctx)[i0] = f32_to_bf16(et);
        static_cast<uint16_t*>(a.ctx)[i1] = f32_to_bf16(ey);
      } else {
        static_cast<float*>(a.ctx)[i0] = et;
        static_cast<float*>(a.ctx)[i1] = ey;
      }
    }
  }
}

cudaError_t launch_condition(const CondArgs& a, cudaStream_t st) {
  if ((a.freq % 4) != 0 || (a.d % 4) != 0) return cudaErrorInvalidValue;
  const size_t smem_h = cond_smem_bytes(a.freq);
  const size_t smem_o = cond_smem_bytes(a.d);
  static bool attr_done[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {  // the largest stage the library's limits allow (d, freq_dim <= 1536)
    const int mx = static_cast<int>(cond_smem_bytes(1536));
    cudaError_t e = cudaFuncSetAttribute(cond_hidden_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(cond_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  if (a.freq > 1536 || a.d > 1536) return cudaErrorInvalidValue;
  const int n = a.R * a.freq;
  cudaError_t e = launch_kernel(cond_sinusoid_kernel, dim3((n + 255) / 256), dim3(256), 0, st, a.t, a.B, a.R, a.freq,
                                 a.t_scale, a.E);
  if (e != cudaSuccess) return e;
  const int rg = (a.R + kCondRows - 1) / kCondRows;
  const dim3 grid((a.d + kCondFeat - 1) / kCondFeat, rg);
  e = launch_kernel(cond_hidden_kernel, grid, dim3(kCondWarps * 32), smem_h, st, (const float*)a.E, a.w1, a.b1, a.hid,
                    a.R, a.freq, a.d);
  if (e != cudaSuccess) return e;
  return launch_kernel(cond_out_kernel, grid, dim3(kCondWarps * 32), smem_o, st, a);
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
      a.h[(static_cast<size_t>(r) * (a.Trow ? a.Trow : T) + a.tok0 + tau0 + t) * a.d + j] = v;
    }
  }
}

// Tiled path: a block computes 32 tokens (of the B unique samples) x 128 output features.
// The tokens' patch vectors and the block's slice of the transposed weights [Kp, d] are
// staged in shared memory in K-chunks of 32; each thread accumulates 4 features x 4 tokens
// (one 16-byte weight load and four broadcast patch loads per 16 multiply-adds), then adds
// bias and position and stores 16-byte groups to row b and, when guided, to row B + b.
constexpr int kPeTok = 32, kPeFeat = 128, kPeK = 32;
__global__ void __launch_bounds__(256) patch_embed_tiled_kernel(PatchArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sx[kPeK][kPeTok + 1];        // patch element k of token t
  __shared__ __align__(16) float sw[kPeK][kPeFeat];  // weight (k, feature)
  const int gh = a.H / a.ph, gw = a.W / a.pw, gf = a.F / a.pt;
  const int T = gf * gh * gw;
  const int Kp = a.C * a.pt * a.ph * a.pw;
  __shared__ int tok_off[kPeTok];   // offset in x of each token's patch corner (-1: past the end)
  __shared__ int k_off[kPeK];       // offset of each patch element from the corner
  const int units = a.B * T;        // the launcher checks that x and the unit count fit 31 bits
  const int u0 = blockIdx.x * kPeTok;
  const int f0 = blockIdx.y * kPeFeat;
  const int fq = threadIdx.x & 31;   // feature quad: features f0 + 4 fq .. + 3
  const int tq = threadIdx.x >> 5;   // token quad: tokens u0 + 4 tq .. + 3
  if (threadIdx.x < kPeTok) {
    const int u = u0 + threadIdx.x;
    int off = -1;
    if (u < units) {
      const int b = u / T, tau = u - b * T;
      const int f = tau / (gh * gw), ii = (tau / gw) % gh, jj = tau % gw;
      off = ((b * a.C * a.F + f * a.pt) * a.H + ii * a.ph) * a.W + jj * a.pw;
    }
    tok_off[threadIdx.x] = off;
  }
  float4 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k0 = 0; k0 < Kp; k0 += kPeK) {
    const int kn = min(kPeK, Kp - k0);
    __syncthreads();
    if (threadIdx.x < kPeK) {
      const int k = k0 + threadIdx.x;
      const int iw = k % a.pw, ih = (k / a.pw) % a.ph, it = (k / (a.pw * a.ph)) % a.pt, c = k / (a.pw * a.ph * a.pt);
      k_off[threadIdx.x] = ((c * a.F + it) * a.H + ih) * a.W + iw;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kPeK * kPeTok; i += blockDim.x) {  // gather patch elements
      const int t = i >> 5, kk = i & 31;  // kPeK == 32
      const int to = tok_off[t];
      sx[kk][t] = (kk < kn && to >= 0) ? __ldg(a.x + to + k_off[kk]) : 0.f;
    }
    for (int i = threadIdx.x; i < kPeK * (kPeFeat / 4); i += blockDim.x) {  // weight slice
      const int kk = i / (kPeFeat / 4), q = i - kk * (kPeFeat / 4);
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      if (kk < kn && f0 + 4 * q < a.d)
        w = __ldg(reinterpret_cast<const float4*>(a.wt + static_cast<size_t>(k0 + kk) * a.d + f0) + q);
      reinterpret_cast<float4*>(&sw[kk][0])[q] = w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kn; ++kk) {
      const float4 w = reinterpret_cast<const float4*>(&sw[kk][0])[fq];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float xv = sx[kk][4 * tq + i];
        acc[i].x = fmaf(xv, w.x, acc[i].x);
        acc[i].y = fmaf(xv, w.y, acc[i].y);
        acc[i].z = fmaf(xv, w.z, acc[i].z);
        acc[i].w = fmaf(xv, w.w, acc[i].w);
      }
    }
  }
  const int f = f0 + 4 * fq;
  if (f >= a.d) return;
  const int Tr = a.Trow ? a.Trow : T;
  const float4 bb = __ldg(reinterpret_cast<const float4*>(a.b + f));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int u = u0 + 4 * tq + i;
    if (u >= units) break;
    const int b = u / T, tau = u - b * T;
    float4 v = make_float4(acc[i].x + bb.x, acc[i].y + bb.y, acc[i].z + bb.z, acc[i].w + bb.w);
    if (a.pos) {
      const float4 pp = __ldg(reinterpret_cast<const float4*>(a.pos + static_cast<size_t>(tau) * a.d + f));
      v.x += pp.x;
      v.y += pp.y;
      v.z += pp.z;
      v.w += pp.w;
    }
    *reinterpret_cast<float4*>(a.h + (static_cast<size_t>(b) * Tr + a.tok0 + tau) * a.d + f) = v;
    if (a.R > a.B) *reinterpret_cast<float4*>(a.h + (static_cast<size_t>(b + a.B) * Tr + a.tok0 + tau) * a.d + f) = v;
  }
}

cudaError_t launch_patch_embed(const PatchArgs& a, cudaStream_t st) {
  const int T = (a.F / a.pt) * (a.H / a.ph) * (a.W / a.pw);
  const int Kp = a.C * a.pt * a.ph * a.pw;
  const long long xsize = static_cast<long long>(a.B) * a.C * a.F * a.H * a.W;
  if (a.wt != nullptr && (a.d & 3) == 0 && (a.R == a.B || a.R == 2 * a.B) && xsize < (1LL << 31)) {
    const long long units = static_cast<long long>(a.B) * T;
    const dim3 grid(static_cast<unsigned>((units + kPeTok - 1) / kPeTok), (a.d + kPeFeat - 1) / kPeFeat);
    if (units == 0) return cudaSuccess;
    return launch_kernel(patch_embed_tiled_kernel, grid, dim3(256), 0, st, a);
  }
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
// A block of 256 threads owns 32 consecutive token rows, so its rows come from at most two
// sample rows r (when T >= 32); the (shift, scale) vectors of those are staged once in shared
// memory instead of being re-read for every token.  Each warp normalises 4 rows, two at a
// time: both rows' float4 loads are in flight before any use, mean and variance are two
// exact passes over registers, and u leaves as 8-byte (bf16), 16-byte (f32) or 4-byte (E4M3)
// stores per lane.  Bound by the memory system: 6 bytes per element for the bf16 output.
constexpr int kLnMaxVec = 12;   // d <= 1536 (float4 per lane)
constexpr int kLnRows = 32;     // token rows per block
constexpr int kLnThreads = 256;
constexpr int kLnWarpRows = kLnRows / (kLnThreads / 32);  // rows per warp, taken two at a time
static_assert(kLnWarpRows % 2 == 0, "a warp normalises its rows in pairs");

// Writes the modulated row; the normalised values replace x (the E4M3 output needs them twice).
template <int OUT, int VEC>
__device__ __forceinline__ void ln_store_row(const LnArgs& a, int m, int lane, int nv, float4 (&x)[VEC], float mean,
                                             float rstd, const float* sh, const float* sc) {
  float amax = 0.f, ss = 0.f;
  float4(&o)[VEC] = x;
#pragma unroll
  for (int k = 0; k < VEC; ++k) {
    const int c = lane + 32 * k;
    if (c < nv) {
      const float4 s4 = reinterpret_cast<const float4*>(sc)[c], b4 = reinterpret_cast<const float4*>(sh)[c];
      o[k].x = (x[k].x - mean) * rstd * (1.f + s4.x) + b4.x;
      o[k].y = (x[k].y - mean) * rstd * (1.f + s4.y) + b4.y;
      o[k].z = (x[k].z - mean) * rstd * (1.f + s4.z) + b4.z;
      o[k].w = (x[k].w - mean) * rstd * (1.f + s4.w) + b4.w;
      if (OUT == 1) {
        uint2 p;
        p.x = pack_bf16x2(o[k].x, o[k].y);
        p.y = pack_bf16x2(o[k].z, o[k].w);
        reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.u) + static_cast<size_t>(m) * a.d)[c] = p;
      } else if (OUT == 0) {
        reinterpret_cast<float4*>(static_cast<float*>(a.u) + static_cast<size_t>(m) * a.d)[c] = o[k];
      } else {
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(o[k].x), fabsf(o[k].y)), fmaxf(fabsf(o[k].z), fabsf(o[k].w))));
        ss += (o[k].x * o[k].x + o[k].y * o[k].y) + (o[k].z * o[k].z + o[k].w * o[k].w);
      }
    }
  }
  if (OUT == 2) {  // E4M3 with the row's scale, and the bound-based scale of the next GELU output
    amax = warp_max(amax);
    ss = warp_sum(ss);
    const float su = amax > 0.f ? amax * (1.0f / 448.0f) : 1.0f;
    const float bound = sqrtf(ss) * a.g_w + a.g_b;
    const float inv = 1.0f / su;
    if (lane == 0) {
      a.su[m] = su;
      a.sg[m] = bound > 0.f ? bound * (1.0f / 448.0f) : 1.0f;
    }
    uint32_t* u8 = reinterpret_cast<uint32_t*>(a.u8 + static_cast<size_t>(m) * a.d);
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
      const int c = lane + 32 * k;
      if (c < nv) u8[c] = pack_e4m3x4(o[k].x * inv, o[k].y * inv, o[k].z * inv, o[k].w * inv);
    }
  }
}

template <int VEC>
__device__ __forceinline__ void ln_load_row(const float* h, int lane, int nv, float4 (&x)[VEC]) {
  const float4* hp = reinterpret_cast<const float4*>(h);
#pragma unroll
  for (int k = 0; k < VEC; ++k) {
    const int c = lane + 32 * k;
    x[k] = c < nv ? hp[c] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

template <int VEC>
__device__ __forceinline__ void ln_stats(const float4 (&x)[VEC], int lane, int nv, int d, float& mean, float& rstd) {
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < VEC; ++k) sum += (x[k].x + x[k].y) + (x[k].z + x[k].w);
  mean = warp_sum(sum) / d;
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < VEC; ++k) {
    const int c = lane + 32 * k;
    if (c < nv) {
      const float dx = x[k].x - mean, dy = x[k].y - mean, dz = x[k].z - mean, dw = x[k].w - mean;
      q += (dx * dx + dy * dy) + (dz * dz + dw * dw);
    }
  }
  rstd = rsqrtf(warp_sum(q) / d + 1e-6f);
}

// OUT: 0 float32, 1 bf16, 2 FP8 E4M3 with the row's scales (see LnArgs).  VEC: float4 per lane
// per row (the smallest of 3, 6, 9, 12 that covers d / 4), so a row takes no more registers
// than it needs.  Each warp's first two rows are requested before the block stages its
// modulation vectors, so the two loads' latencies overlap.
template <int OUT, int VEC>
__global__ void __launch_bounds__(kLnThreads) ln_modulate_kernel(LnArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float ln_mod[];  // [2 sample rows][shift | scale][d]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = a.d >> 2;
  const int m0 = blockIdx.x * kLnRows;
  float4 xa[VEC], xb[VEC];
  {
    const int ma = m0 + warp * kLnWarpRows, mb = ma + 1;
    if (ma < a.M) ln_load_row<VEC>(a.h + static_cast<size_t>(ma) * a.d, lane, nv, xa);
    if (mb < a.M) ln_load_row<VEC>(a.h + static_cast<size_t>(mb) * a.d, lane, nv, xb);
  }
  // sample rows of this block's first and last token rows; staged when at most two
  const int rfirst = a.ld_mod ? m0 / a.T : 0;
  const int rlast = a.ld_mod ? min(m0 + kLnRows - 1, a.M - 1) / a.T : 0;
  const bool staged = rlast - rfirst <= 1;
  if (staged) {
    for (int i = threadIdx.x; i < (rlast - rfirst + 1) * nv; i += blockDim.x) {
      const int j = i / nv, c = i - j * nv;
      const size_t off = static_cast<size_t>(rfirst + j) * a.ld_mod;
      reinterpret_cast<float4*>(ln_mod + (2 * j) * a.d)[c] = __ldg(reinterpret_cast<const float4*>(a.shift + off) + c);
      reinterpret_cast<float4*>(ln_mod + (2 * j + 1) * a.d)[c] = __ldg(reinterpret_cast<const float4*>(a.scale + off) + c);
    }
  }
  __syncthreads();
  for (int pr = 0; pr < kLnWarpRows; pr += 2) {  // each warp: rows m0 + kLnWarpRows warp + {0, 1}, {2, 3}, ...
    const int ma = m0 + warp * kLnWarpRows + pr, mb = ma + 1;
    if (ma >= a.M) break;
    const bool hb = mb < a.M;
    if (pr > 0) {
      ln_load_row<VEC>(a.h + static_cast<size_t>(ma) * a.d, lane, nv, xa);
      if (hb) ln_load_row<VEC>(a.h + static_cast<size_t>(mb) * a.d, lane, nv, xb);
    }
    float mean, rstd;
    ln_stats<VEC>(xa, lane, nv, a.d, mean, rstd);
    {
      const int r = a.ld_mod ? ma / a.T : 0;
      const float* sh = staged ? ln_mod + 2 * (r - rfirst) * a.d : a.shift + static_cast<size_t>(r) * a.ld_mod;
      const float* sc = staged ? ln_mod + (2 * (r - rfirst) + 1) * a.d : a.scale + static_cast<size_t>(r) * a.ld_mod;
      ln_store_row<OUT, VEC>(a, ma, lane, nv, xa, mean, rstd, sh, sc);
    }
    if (hb) {
      ln_stats<VEC>(xb, lane, nv, a.d, mean, rstd);
      const int r = a.ld_mod ? mb / a.T : 0;
      const float* sh = staged ? ln_mod + 2 * (r - rfirst) * a.d : a.shift + static_cast<size_t>(r) * a.ld_mod;
      const float* sc = staged ? ln_mod + (2 * (r - rfirst) + 1) * a.d : a.scale + static_cast<size_t>(r) * a.ld_mod;
      ln_store_row<OUT, VEC>(a, mb, lane, nv, xb, mean, rstd, sh, sc);
    }
  }
}

template <int VEC>
static cudaError_t launch_ln_vec(const LnArgs& a, int grid, size_t smem, cudaStream_t st) {
  if (a.u8 != nullptr) return launch_kernel(ln_modulate_kernel<2, VEC>, dim3(grid), dim3(kLnThreads), smem, st, a);
  if (a.u_bf16) return launch_kernel(ln_modulate_kernel<1, VEC>, dim3(grid), dim3(kLnThreads), smem, st, a);
  return launch_kernel(ln_modulate_kernel<0, VEC>, dim3(grid), dim3(kLnThreads), smem, st, a);
}

cudaError_t launch_ln_modulate(const LnArgs& a, cudaStream_t st) {
  if ((a.d & 3) != 0 || a.d > 4 * 32 * kLnMaxVec) return cudaErrorInvalidValue;
  const int grid = (a.M + kLnRows - 1) / kLnRows;
  if (grid == 0) return cudaSuccess;
  if (a.u8 != nullptr && (a.su == nullptr || a.sg == nullptr)) return cudaErrorInvalidValue;
  const size_t smem = 4 * static_cast<size_t>(a.d) * sizeof(float);
  const int nv = a.d >> 2;
  if (nv <= 32 * 3) return launch_ln_vec<3>(a, grid, smem, st);
  if (nv <= 32 * 6) return launch_ln_vec<6>(a, grid, smem, st);
  if (nv <= 32 * 9) return launch_ln_vec<9>(a, grid, smem, st);
  return launch_ln_vec<12>(a, grid, smem, st);
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

// ============================================================================ guidance + unpatchify
// One thread per output element of [B, Cout, F, H, W], in memory order (stores coalesced);
// the two decoder values it combines sit in rows b and B + b of z at the element's token.
__global__ void __launch_bounds__(256) cfg_unpatchify_kernel(UnpatchArgs a) {
  pdl_trigger();
  pdl_wait();
  const long long total = static_cast<long long>(a.B) * a.Cout * a.F * a.H * a.W;
  const int gh = a.H / a.ph, gw = a.W / a.pw;
  for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    long long r = idx;
    const int ww = static_cast<int>(r % a.W);
    r /= a.W;
    const int hh = static_cast<int>(r % a.H);
    r /= a.H;
    const int fr = static_cast<int>(r % a.F);
    r /= a.F;
    const int c = static_cast<int>(r % a.Cout);
    const int b = static_cast<int>(r / a.Cout);
    const int tau = ((fr / a.pt) * gh + hh / a.ph) * gw + ww / a.pw;
    const int p = (((fr % a.pt) * a.ph + hh % a.ph) * a.pw + ww % a.pw) * a.Cout + c;
    const int Tr = a.Trow ? a.Trow : a.T;
    const float zc = __ldg(a.z + (static_cast<size_t>(b) * Tr + a.tok0 + tau) * a.P + p);
    float v = zc;
    if (a.guided && (a.gch <= 0 || c < a.gch)) {
      const float zu = __ldg(a.z + (static_cast<size_t>(b + a.B) * Tr + a.tok0 + tau) * a.P + p);
      v = zu + a.s * (zc - zu);
    }
    a.out[idx] = v;
  }
}

cudaError_t launch_cfg_unpatchify(const UnpatchArgs& a, int num_sms, cudaStream_t st) {
  const long long total = static_cast<long long>(a.B) * a.Cout * a.F * a.H * a.W;
  if (total == 0) return cudaSuccess;
  const long long want = (total + 255) / 256;
  const int grid = static_cast<int>(want < 8LL * num_sms ? want : 8LL * num_sms);
  return launch_kernel(cfg_unpatchify_kernel, dim3(grid), dim3(256), 0, st, a);
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
__global__ void pos_tables_kernel(float* pos, float* rope, int gf, int gh, int gw, int d, int dh, int tok0) {
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
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < (T + tok0) * (dh / 2); idx += gridDim.x * blockDim.x) {
      const int row = idx / (dh / 2), i = idx - row * (dh / 2);
      if (row < tok0) {  // condition tokens: no rotation
        rope[2 * idx] = 1.f;
        rope[2 * idx + 1] = 0.f;
        continue;
      }
      const int tau = row - tok0;
      const int axis = (2 * i) / sl, k = ((2 * i) % sl) / 2;
      const int coord = axis == 0 ? tau / (gh * gw) : (axis == 1 ? (tau / gw) % gh : tau % gw);
      const double ang = coord * pow(10000.0, -2.0 * k / sl);
      rope[2 * idx] = static_cast<float>(cos(ang));
      rope[2 * idx + 1] = static_cast<float>(sin(ang));
    }
  }
}

cudaError_t launch_pos_tables(float* pos, float* rope, int gf, int gh, int gw, int d, int dh, int tok0,
                              cudaStream_t st) {
  pos_tables_kernel<<<256, 256, 0, st>>>(pos, rope, gf, gh, gw, d, dh, tok0);
  return cudaGetLastError();
}

// ============================================================================ f32 cross-attention
// One warp per (token, head): lanes split the head dim for the two scores, then write the
// softmax mix of the two condition values.
__global__ void xattn_f32_kernel(XAttnArgs a) {
  pdl_trigger();
  pdl_wait();
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<long long>(a.M) * a.H) return;
  const int m = static_cast<int>(w / a.H), head = static_cast<int>(w - static_cast<long long>(m) * a.H);
  const int row = m / a.T;
  const float* q = a.q + static_cast<size_t>(m) * a.d + head * a.dh;
  const float* k0 = a.xkv + static_cast<size_t>(2 * row) * a.ld_xkv + head * a.dh;
  const float* k1 = k0 + a.ld_xkv;
  float s0 = 0.f, s1 = 0.f;
  for (int j = lane; j < a.dh; j += 32) {
    s0 = fmaf(q[j], k0[j], s0);
    s1 = fmaf(q[j], k1[j], s1);
  }
  const float sc = rsqrtf(static_cast<float>(a.dh));
  s0 = warp_sum(s0) * sc;
  s1 = warp_sum(s1) * sc;
  const float mx = fmaxf(s0, s1);
  const float e0 = expf(s0 - mx), e1 = expf(s1 - mx);
  const float p0 = e0 / (e0 + e1), p1 = e1 / (e0 + e1);
  float* o = a.o + static_cast<size_t>(m) * a.d + head * a.dh;
  for (int j = lane; j < a.dh; j += 32) o[j] = p0 * k0[a.d + j] + p1 * k1[a.d + j];
}

cudaError_t launch_xattn_f32(const XAttnArgs& a, cudaStream_t st) {
  const long long warps = static_cast<long long>(a.M) * a.H;
  if (warps == 0) return cudaSuccess;
  return launch_kernel(xattn_f32_kernel, dim3(static_cast<unsigned>((warps + 7) / 8)), dim3(256), 0, st, a);
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

// One block per row: the row's largest magnitude, then every element divided by amax / 448
// and rounded to E4M3 (cols % 4 == 0).
__global__ void __launch_bounds__(256) quantize_rows_e4m3_kernel(const float* __restrict__ src, uint8_t* __restrict__ dst,
                                                                 float* __restrict__ scale, int cols) {
  __shared__ float red[8];
  const float4* row = reinterpret_cast<const float4*>(src + static_cast<size_t>(blockIdx.x) * cols);
  const int n4 = cols / 4;
  float m = 0.f;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = row[i];
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_max(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float s = red[0] > 0.f ? red[0] * (1.0f / 448.0f) : 1.0f;
  if (threadIdx.x == 0) scale[blockIdx.x] = s;
  const float inv = 1.0f / s;
  uint32_t* out = reinterpret_cast<uint32_t*>(dst + static_cast<size_t>(blockIdx.x) * cols);
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = row[i];
    out[i] = pack_e4m3x4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
  }
}

cudaError_t launch_quantize_rows_e4m3(const float* src, uint8_t* dst, float* scale, int rows, int cols,
                                      cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (cols % 4) return cudaErrorInvalidValue;
  quantize_rows_e4m3_kernel<<<rows, 256, 0, st>>>(src, dst, scale, cols);
  return cudaGetLastError();
}

// bf16 rows -> E4M3 with a per-row scale amax / 448 (1 for an all-zero row), one warp per row:
// the forward's attention output before the FP8 out-projection.  Each lane keeps its share of
// the row (groups of 4) in registers between the amax and the conversion.
constexpr int kQ8MaxVec = 12;  // d <= 1536
__global__ void __launch_bounds__(256) quantize_rows_bf16_e4m3_kernel(const uint16_t* __restrict__ src,
                                                                      uint8_t* __restrict__ dst,
                                                                      float* __restrict__ scale, int rows, int cols) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int n4 = cols >> 2;
  const uint2* in = reinterpret_cast<const uint2*>(src + static_cast<size_t>(row) * cols);
  float4 v[kQ8MaxVec];
  float m = 0.f;
#pragma unroll
  for (int k = 0; k < kQ8MaxVec; ++k) {
    const int c = lane + 32 * k;
    if (c < n4) {
      const uint2 p = in[c];
      v[k] = make_float4(bf16_to_f32(static_cast<uint16_t>(p.x & 0xffffu)), bf16_to_f32(static_cast<uint16_t>(p.x >> 16)),
                         bf16_to_f32(static_cast<uint16_t>(p.y & 0xffffu)), bf16_to_f32(static_cast<uint16_t>(p.y >> 16)));
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v[k].x), fabsf(v[k].y)), fmaxf(fabsf(v[k].z), fabsf(v[k].w))));
    }
  }
  m = warp_max(m);
  const float s = m > 0.f ? m * (1.0f / 448.0f) : 1.0f;
  if (lane == 0) scale[row] = s;
  const float inv = 1.0f / s;
  uint32_t* out = reinterpret_cast<uint32_t*>(dst + static_cast<size_t>(row) * cols);
#pragma unroll
  for (int k = 0; k < kQ8MaxVec; ++k) {
    const int c = lane + 32 * k;
    if (c < n4) out[c] = pack_e4m3x4(v[k].x * inv, v[k].y * inv, v[k].z * inv, v[k].w * inv);
  }
}

cudaError_t launch_quantize_rows_bf16_e4m3(const uint16_t* src, uint8_t* dst, float* scale, int rows, int cols,
                                           cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (cols % 4 || cols > 4 * 32 * kQ8MaxVec) return cudaErrorInvalidValue;
  return launch_kernel(quantize_rows_bf16_e4m3_kernel, dim3((rows + 7) / 8), dim3(256), 0, st, src, dst, scale, rows,
                       cols);
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
