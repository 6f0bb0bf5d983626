// Internal launch interfaces between the C-ABI layer (dit_api.cu) and the kernel
// translation units.  Plain structs of device pointers and sizes.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dit {

// ------------------------------------------------------------------ GEMM epilogues
enum Epi : int {
  EPI_F32 = 0,    // out[m, n] = acc + bias[n]                              (float32)
  EPI_ADALN = 1,  // out[n, m] = acc + bias[m]   (A = modulation weights, B = SiLU(c) rows)
  EPI_GELU = 2,   // out[m, n] = gelu_tanh(acc + bias[n])                   (bf16 / f32)
  EPI_RESID = 3,  // h[m, n]  += gate[row(m), n] * (acc + bias[n])          (float32 RMW, direct)
  EPI_QKV = 4,       // scatter to q, k, v head-major, column by column
  EPI_QKV_HEAD = 5,  // same, one whole head at a time (+ QK-RMSNorm, 3D RoPE); tile = 2 heads
  // Swapped operands (A = weights, B = activations: GEMM rows are output features,
  // GEMM columns are tokens; ea.M = features, ea.N = tokens):
  EPI_RESID_T = 6,   // h[tok, f] += gate[row(tok), f] * (acc + bias[f])   (TMA reduce-add)
  EPI_QKV_T = 7,     // q, k, v^T scatter, 32 x 32 chunks staged through shared memory
  // Cross-attention onto a two-token condition sequence, fused into the query projection:
  // tile = 2 heads; each thread holds one token's query for one head, scores it against the
  // two keys, and writes the softmax mix of the two values to o [M, d] (bf16).
  EPI_XATTN = 8,
  // FP8 E4M3 operands (kind::f8f6f4): the accumulator is scaled by the per-row scale sa[m] of
  // the A operand and the per-column scale sb[n] of the B operand before the epilogue proper.
  EPI_F32_8 = 9,     // out[m, n] = sa[m] sb[n] acc + bias[n]                  (float32)
  EPI_GELU8 = 10,    // g = gelu(sa[m] sb[n] acc + bias[n]) stored as E4M3 g / sg[m] (bytes [M, ldo])
  EPI_RESID_T8 = 11, // swapped: h[tok, f] += gate * (sa[f] sb[tok] acc + bias[f]) (TMA reduce-add)
  EPI_QKV_T8 = 12,   // swapped q, k, v^T scatter of sa[f] sb[tok] acc + bias[f]
  EPI_QKV_HEAD8 = 13,  // whole-head scatter (+ QK-RMSNorm, 3D RoPE) of sa[m] sb[n] acc + bias[n]
};
template <int EPI>
__host__ __device__ constexpr bool epi_fp8() {
  return EPI == EPI_F32_8 || EPI == EPI_GELU8 || EPI == EPI_RESID_T8 || EPI == EPI_QKV_T8 || EPI == EPI_QKV_HEAD8;
}

struct EpiArgs {
  int M, N;             // logical output extent (rows of A, rows of B)
  const float* bias;    // [N], or [M] for EPI_ADALN
  void* out;            // EPI_F32 / EPI_ADALN / EPI_GELU destination
  int ldo;              // its row stride in elements
  // EPI_RESID
  float* h;             // residual stream [M, ldh]
  int ldh;
  const float* gate;    // gate vector of row r at gate + r * ld_gate
  int ld_gate;
  int T;                // tokens per sample (row(m) = m / T)
  // EPI_QKV
  void* q;              // bf16 [R*H, Tpad, DP]  (f32 path: [R*H, T, dh])
  void* k;
  void* v;              // bf16 transposed [R*H, DP, Tpad] (f32 path: [R*H, T, dh])
  int d, H, dh, DP, Tpad;
  const float* qn;      // [dh] RMSNorm gains or nullptr
  const float* kn;
  const float* rope;    // [T, dh/2, 2] (cos, sin) or nullptr
  // EPI_XATTN: keys and values of the condition tokens of row r at
  // xkv + (2r + s) * ld_xkv + {0: k, d: v} + head * dh (s = 0, 1), float32
  const float* xkv;
  int ld_xkv;
  void* xo;             // bf16 [M, d] attention output
  // FP8 operand scales (per A row, per B row) and the E4M3 output scale of EPI_GELU8
  const float* sa;
  const float* sb;
  const float* sg;
  // EPI_RESID_T / EPI_RESID_T8: split K into this many slices (each adds its partial product
  // into the residual stream; 0 or 1 = no split)
  int ksplit;
  int* status;
};

// tensor-core GEMM D[M, N] = A[M, K] B[N, K]^T with A, B bf16 K-major.
// Returns cudaSuccess or the launch error.
// EPI_RESID_T / EPI_RESID_T8 update the residual stream through shared memory with a TMA
// reduce-add: tmC maps the float32 stream [tokens, features], box 16 tokens x 32 features,
// 128B swizzle.  Other epilogues ignore tmC.
cudaError_t launch_gemm_tc(int epi, int block_n, const CUtensorMap* tmA, const CUtensorMap* tmB, int K,
                           const EpiArgs& ea, int num_sms, cudaStream_t st, const CUtensorMap* tmC = nullptr);
int gemm_tc_supported_bn(int block_n);
// Same GEMM on SM pairs (cluster of 2, tcgen05 cta_group::2): 256 x block_n tiles;
// tmA box = 128 rows x 64, tmB box = block_n/2 rows x 64.
cudaError_t launch_gemm_tc2(int epi, int block_n, const CUtensorMap* tmA, const CUtensorMap* tmB, int K,
                            const EpiArgs& ea, int num_sms, cudaStream_t st, const CUtensorMap* tmC = nullptr);
int gemm_tc2_supported_bn(int block_n);
// Build a 2-D bf16 K-major tensor map: rows x K, box = box_rows x 64, 128-byte swizzle.
// Per-device one-time launch set-up (a kernel's shared-memory attribute is set on the
// current device): index of the current device, or -1 if there is none or it is beyond
// kMaxDevices.
constexpr int kMaxDevices = 64;
inline int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}
bool make_tmap_bf16_kmajor(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows);
// FP8 (one byte per element) K-major map: rows x K, box = box_rows x 128, 128-byte swizzle.
bool make_tmap_e4m3_kmajor(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows);
// 3-d bf16 map: dims d0 (innermost) x d1 x d2, box box0 x box1 x 1, 128B swizzle or none.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0,
                       uint32_t box1, int swizzle_bytes);
// General 2-D bf16 tensor map: rows x cols (cols contiguous), box box_rows x box_cols,
// swizzle 128 / 64 / 32 bytes (0 = none).  The box row (box_cols * 2 bytes) must not
// exceed the swizzle span.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                    uint32_t box_rows, int swizzle_bytes);
// Same for a float32 matrix.
bool make_tmap_f32(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                   uint32_t box_rows, int swizzle_bytes);

// float32 SIMT GEMM with the same epilogues (f32 outputs everywhere).
cudaError_t launch_gemm_simt(int epi, const float* A, const float* B, int M, int N, int K, const EpiArgs& ea,
                             cudaStream_t st);

// ------------------------------------------------------------------ small steps
struct CondArgs {
  const float* t;        // [B]
  const void* y;         // int32 [B] or float32 [B, d]
  int B, R, d, freq, cond_kind, num_classes, guided;
  float t_scale;
  const float *w1, *b1, *w2, *b2, *table;
  float* E;              // scratch [R, freq]
  float* hid;            // scratch [R, d]
  float* c;              // [R, d]   (optional, may be null)
  void* sc;              // SiLU(c): bf16 [*, d] or f32 [R, d] (optional, may be null)
  int sc_bf16;
  int* status;
  // the two condition embeddings e_t (timestep MLP) and e_y (label row / text vector) as
  // tokens: in the residual stream at tok_h + r * tok_ld (e_t) and + d (e_y), and / or as
  // rows 2r, 2r + 1 of a condition sequence ctx [2R, d] (bf16 or f32)
  float* tok_h = nullptr;
  size_t tok_ld = 0;
  void* ctx = nullptr;
  int ctx_bf16 = 0;
};
cudaError_t launch_condition(const CondArgs& a, cudaStream_t st);

struct PatchArgs {
  const float* x;        // [B, C, F, H, W]
  const float* w;        // [d, Kp]
  const float* wt;       // the same weights transposed, [Kp, d]
  const float* b;        // [d]
  const float* pos;      // [T, d] or nullptr
  float* h;              // [R*Trow, d]: patch token tau of row r at row r * Trow + tok0 + tau
  int B, R, C, F, H, W, pt, ph, pw, d;
  int Trow = 0, tok0 = 0;  // tokens per row in h (0: the patch count) and the first patch token
};
cudaError_t launch_patch_embed(const PatchArgs& a, cudaStream_t st);

struct LnArgs {
  const float* h;        // [M, d]
  void* u;               // bf16 or f32 [M, d] (E4M3 bytes when u8 is set)
  int u_bf16;
  // FP8 output: u as E4M3 with a per-row scale su[m] = amax_m / 448, and the per-row scale
  // sg[m] = (||u_m||_2 * g_w + g_b) / 448 of the next matmul's GELU output (a bound on it)
  uint8_t* u8 = nullptr;
  float* su = nullptr;
  float* sg = nullptr;
  float g_w = 0.f, g_b = 0.f;
  const float* shift;    // row r vector at shift + r * ld_mod
  const float* scale;
  int ld_mod;
  int M, T, d;
};
cudaError_t launch_ln_modulate(const LnArgs& a, cudaStream_t st);

struct AttnArgs {
  const void *q, *k, *v;  // layouts as in EpiArgs (bf16 head-major padded or f32 head-major)
  void* o;                // [R*T, d] bf16 or f32, token-major
  int R, H, T, dh, DP, Tpad, d;
  int bf16;               // 1: bf16 padded layouts, V transposed
};
cudaError_t launch_attention_simt(const AttnArgs& a, cudaStream_t st);
// Tensor maps of the tensor-core attention: q / k main (box 128 x 64, 128B swizzle),
// q / k tail (head-dim columns 64..79, box 128 x 16, 32B swizzle; unused when dh = 64),
// v (transposed, box DP x 64, 128B swizzle), o (output [R][T][d] as a 3-d map, box dh x 128 x 1,
// so rows past T are clipped).
struct AttnMaps {
  CUtensorMap q, qt, k, kt, v, o;
};
bool make_attention_maps(AttnMaps* m, const void* q, const void* k, const void* v, void* o, int R, int H, int T,
                         int Tpad, int dh, int DP, int d);
cudaError_t launch_attention_tc(const AttnArgs& a, const AttnMaps& maps, int* status, cudaStream_t st);

struct QkNormArgs {   // f32 path: RMSNorm + RoPE applied in place to q, k [R*H, T, dh]
  float *q, *k;
  const float *qn, *kn, *rope;
  int RH, T, dh;
};
cudaError_t launch_qknorm_rope_f32(const QkNormArgs& a, cudaStream_t st);

// Classifier-free guidance combine and unpatchify of the decoder output z:
// out[b, c, f*pt+it, i*ph+ih, j*pw+iw] = z_null + s (z_cond - z_null) at token (f, i, j) and
// vector index ((it*ph + ih)*pw + iw)*Cout + c (z_cond alone when not guided, and on channels
// c >= gch when gch > 0).
struct UnpatchArgs {
  const float* z;        // [R*Trow, P], rows [cond; uncond] when guided; patch token tau of row r
                         // at row r * Trow + tok0 + tau
  float* out;            // [B, Cout, F, H, W]
  int B, T, P, Cout, F, H, W, pt, ph, pw, guided;
  int gch;               // guided channels: c < gch are guided, the rest keep z_cond (0: all)
  float s;
  int Trow = 0, tok0 = 0;
};
cudaError_t launch_cfg_unpatchify(const UnpatchArgs& a, int num_sms, cudaStream_t st);

// Sampler update x_next = c0 * x + c1 * pred, pred = the first n_sample values of each
// sample's ld_pred-long block of the denoiser output (its first C channels).
struct SamplerArgs {
  const float* x;        // [B, n_sample]
  const float* pred;     // [B, ld_pred]
  float* x_next;         // [B, n_sample], may alias x
  long long n_sample, ld_pred;
  int B;
  float c0, c1;
};
cudaError_t launch_sampler_step(const SamplerArgs& a, int num_sms, cudaStream_t st);

// rope rows tok0 .. tok0 + gf*gh*gw - 1 hold the patch tokens' rotations; rows < tok0
// (condition tokens) the identity (cos 1, sin 0)
cudaError_t launch_pos_tables(float* pos, float* rope, int gf, int gh, int gw, int d, int dh, int tok0,
                              cudaStream_t st);

// float32 cross-attention onto the two condition tokens (the fp32 path's unfused form of
// EPI_XATTN): o[m, head] = softmax over s of q[m, head] . k_s / sqrt(dh), mixing v_s.
struct XAttnArgs {
  const float* q;        // [M, d]
  const float* xkv;      // as EpiArgs::xkv
  int ld_xkv;
  float* o;              // [M, d]
  int M, T, d, H, dh;
};
cudaError_t launch_xattn_f32(const XAttnArgs& a, cudaStream_t st);
cudaError_t launch_f32_to_bf16(const float* src, uint16_t* dst, size_t n, cudaStream_t st);
// Row-wise E4M3 quantisation of a float32 matrix [rows, cols]: scale[r] = amax_r / 448 (1 for a
// zero row), dst[r, c] = E4M3(src[r, c] / scale[r]).
cudaError_t launch_quantize_rows_e4m3(const float* src, uint8_t* dst, float* scale, int rows, int cols,
                                      cudaStream_t st);
// bf16 rows [rows, cols] -> E4M3 bytes with per-row scales amax / 448; cols % 4 == 0, <= 1536.
cudaError_t launch_quantize_rows_bf16_e4m3(const uint16_t* src, uint8_t* dst, float* scale, int rows, int cols,
                                           cudaStream_t st);
cudaError_t launch_wait_probe(int* flag, int* status, long long limit_ns, cudaStream_t st);

}  // namespace dit
