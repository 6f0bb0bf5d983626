// C-ABI layer: configuration checks, device weights and workspace, tensor maps,
// and the kernel sequence of one DiT denoiser forward.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"

using namespace dit;

namespace {

struct BlockW {
  void *qkv_w = nullptr, *proj_w = nullptr, *fc1_w = nullptr, *fc2_w = nullptr;  // bf16 or f32
  float *qkv_b = nullptr, *proj_b = nullptr, *fc1_b = nullptr, *fc2_b = nullptr;
  float *qn = nullptr, *kn = nullptr;
  // in-context / cross-attention designs: learned LayerNorm affines, stored as (gain - 1, bias)
  // so that the LN + modulate kernel applies them as a row-independent (scale, shift)
  float *ln1_s = nullptr, *ln1_b = nullptr, *ln2_s = nullptr, *ln2_b = nullptr, *xln_s = nullptr, *xln_b = nullptr;
  // cross-attention: query and output projections (the key / value projections of all blocks
  // are stacked in the handle for one GEMM at the start of the forward)
  void *xq_w = nullptr, *xo_w = nullptr;
  float *xq_b = nullptr, *xo_b = nullptr;
  // FP8 feed-forward: E4M3 weights with per-output-channel scales, and the constants of the
  // hidden activation's scale bound (max_n ||fc1.w_n||_2, max |fc1.b|)
  uint8_t *fc1_w8 = nullptr, *fc2_w8 = nullptr;
  float *fc1_s = nullptr, *fc2_s = nullptr;
  float g_w = 0.f, g_b = 0.f;
  // FP8 attention projections: E4M3 in- and out-projection weights, per-output-channel scales
  uint8_t *qkv_w8 = nullptr, *proj_w8 = nullptr;
  float *qkv_s = nullptr, *proj_s = nullptr;
  CUtensorMap tm_qkv8, ta_qkv8, ta_proj8;  // as the B operand (two-head tiles) / the swapped A operand
  CUtensorMap tm_qkv, tm_fc1, tm_xq, tm_fc1_8;  // weights as the B operand (box = tile width rows)
  CUtensorMap tm_fc1_h;  // fc1 weights as the B operand of the SM-pair GEMM (each CTA loads half: 128 rows)
  CUtensorMap ta_qkv, ta_proj, ta_fc2, ta_xo, ta_fc2_8;  // weights as the A operand of the swapped GEMMs (box 128 rows)
};

struct Geometry {
  int gf, gh, gw, T, Kp, P, Cout, dh, DP, Tpad, Rmax, RPalloc, Mmax, nmod;
  int kind;      // DIT_BLOCK_*
  int Tc, Ts;    // condition tokens in front of the patch tokens; tokens per row inside the blocks
  int mpb;       // modulation vectors per block (6 adaLN-Zero, 4 adaLN, 0 otherwise)
  int nkv;       // cross-attention: key / value features of all blocks (depth * 2d)
  int CTXalloc;  // rows of the condition-sequence buffer (2 Rmax rounded up for 256-row boxes)
  int bn_qkv, bn_fc1;
  int bn_dec, dec_rows;  // decoder GEMM tile width; decoder weight rows (P padded to whole tiles)
  int headwise;  // 1: QK-RMSNorm / RoPE need whole heads -> two-head tiles for the QKV projection
};

bool validate(const dit_config* c, std::string& err) {
  auto bad = [&](const char* m) {
    err = m;
    return false;
  };
  if (c == nullptr) return bad("config is NULL");
  if (c->dtype != DIT_DTYPE_F32 && c->dtype != DIT_DTYPE_BF16) return bad("dtype must be DIT_DTYPE_F32 or DIT_DTYPE_BF16");
  if (c->in_channels <= 0 || c->frames <= 0 || c->height <= 0 || c->width <= 0) return bad("latent extent must be positive");
  if (c->patch_t <= 0 || c->patch_h <= 0 || c->patch_w <= 0) return bad("patch extent must be positive");
  if (c->frames % c->patch_t || c->height % c->patch_h || c->width % c->patch_w)
    return bad("patch extent must divide the latent extent");
  if (c->hidden <= 0 || c->depth < 0 || c->heads <= 0 || c->mlp_hidden <= 0) return bad("model sizes must be positive");
  if (c->hidden % c->heads) return bad("hidden must be a multiple of heads");
  if (c->learn_sigma != 0 && c->learn_sigma != 1) return bad("learn_sigma must be 0 or 1");
  if (c->pos_kind != DIT_POS_SINCOS2D && c->pos_kind != DIT_POS_ROPE3D) return bad("unknown pos_kind");
  if (c->qk_norm != 0 && c->qk_norm != 1) return bad("qk_norm must be 0 or 1");
  if (c->cond_kind != DIT_COND_CLASS && c->cond_kind != DIT_COND_VECTOR) return bad("unknown cond_kind");
  if (c->cond_kind == DIT_COND_CLASS && c->num_classes <= 0) return bad("num_classes must be positive");
  if (c->freq_dim <= 0 || (c->freq_dim & 3)) return bad("freq_dim must be a positive multiple of 4");
  if (c->max_batch <= 0) return bad("max_batch must be positive");
  if (!isfinite(c->t_scale)) return bad("t_scale must be finite");
  if (c->block_kind < DIT_BLOCK_ADALN_ZERO || c->block_kind > DIT_BLOCK_ADALN) return bad("unknown block_kind");
  if (c->ffn_fp8 != 0 && c->ffn_fp8 != 1) return bad("ffn_fp8 must be 0 or 1");
  if (c->attn_fp8 != 0 && c->attn_fp8 != 1) return bad("attn_fp8 must be 0 or 1");
  return true;
}

// Shapes the kernels cover (DIT_ERR_UNSUPPORTED otherwise).
bool supported(const dit_config* c, std::string& err) {
  const int dh = c->hidden / c->heads;
  if (dh != 64 && dh != 72) {
    err = "head dim (hidden / heads) must be 64 or 72";
    return false;
  }
  if (c->hidden % 4 || c->hidden > 1536) {
    err = "hidden must be a multiple of 4 and at most 1536";
    return false;
  }
  if (c->freq_dim > 1536) {
    err = "freq_dim must be at most 1536";
    return false;
  }
  if (c->pos_kind == DIT_POS_SINCOS2D && (c->frames / c->patch_t != 1 || c->hidden % 4)) {
    err = "2D sin-cos positions need one frame of patches and hidden % 4 == 0";
    return false;
  }
  if (c->pos_kind == DIT_POS_ROPE3D && dh % 6) {
    err = "3D RoPE needs head dim % 6 == 0";
    return false;
  }
  if (c->dtype == DIT_DTYPE_BF16) {
    if (c->hidden % (2 * dh) || c->hidden % 32 || c->mlp_hidden % 32) {
      err = "bf16 path needs an even number of heads and hidden, mlp_hidden multiples of 32";
      return false;
    }
  }
  if (c->ffn_fp8 && c->dtype != DIT_DTYPE_BF16) {
    err = "the FP8 feed-forward runs on the bf16 tensor-core path only";
    return false;
  }
  if (c->attn_fp8 && c->dtype != DIT_DTYPE_BF16) {
    err = "the FP8 attention projections run on the bf16 tensor-core path only";
    return false;
  }
  const long long kp = 1LL * c->in_channels * c->patch_t * c->patch_h * c->patch_w;
  if (kp * 16 * 4 > 200 * 1024) {
    err = "patch vector too long";
    return false;
  }
  return true;
}

Geometry geometry(const dit_config* c) {
  Geometry g;
  g.gf = c->frames / c->patch_t;
  g.gh = c->height / c->patch_h;
  g.gw = c->width / c->patch_w;
  g.T = g.gf * g.gh * g.gw;
  g.kind = c->block_kind;
  g.Tc = g.kind == DIT_BLOCK_IN_CONTEXT ? 2 : 0;
  g.Ts = g.T + g.Tc;
  g.mpb = g.kind == DIT_BLOCK_ADALN_ZERO ? 6 : g.kind == DIT_BLOCK_ADALN ? 4 : 0;
  g.Kp = c->in_channels * c->patch_t * c->patch_h * c->patch_w;
  g.Cout = c->learn_sigma ? 2 * c->in_channels : c->in_channels;
  g.P = c->patch_t * c->patch_h * c->patch_w * g.Cout;
  g.dh = c->hidden / c->heads;
  g.DP = (g.dh + 15) / 16 * 16;
  g.Tpad = (g.Ts + 127) / 128 * 128;
  g.Rmax = c->cond_kind == DIT_COND_CLASS ? 2 * c->max_batch : c->max_batch;
  g.RPalloc = (g.Rmax + 255) / 256 * 256;
  g.Mmax = g.Rmax * g.Ts;
  g.nmod = g.mpb > 0 ? (g.mpb * c->depth + 2) * c->hidden : 0;
  g.nkv = g.kind == DIT_BLOCK_CROSS_ATTN ? 2 * c->depth * c->hidden : 0;
  g.CTXalloc = (2 * g.Rmax + 255) / 256 * 256;
  // GEMM tiles.  The MMA reads its A and B tiles from shared memory every instruction,
  // so wide (N = 256) tiles keep the tensor cores fed.  proj, fc2 and (without QK norm
  // / RoPE) QKV run with swapped operands — A = weights (features), B = tokens — so the
  // N = 256 tile runs over tokens and the tile count fills the SMs; fc1 runs directly.
  g.headwise = (c->qk_norm || c->pos_kind == DIT_POS_ROPE3D) ? 1 : 0;
  g.bn_qkv = g.headwise ? 2 * g.dh : 256;
  g.bn_fc1 = 256;
  g.bn_dec = g.P <= 16 ? 16 : g.P <= 32 ? 32 : g.P <= 64 ? 64 : g.P <= 128 ? 128 : 256;
  g.dec_rows = (g.P + g.bn_dec - 1) / g.bn_dec * g.bn_dec;
  return g;
}

int weight_count(const dit_config* c) {
  const int k = c->block_kind;
  const int per_block = (k == DIT_BLOCK_IN_CONTEXT ? 12 : k == DIT_BLOCK_CROSS_ATTN ? 20 : 10) + (c->qk_norm ? 2 : 0);
  return 6 + (c->cond_kind == DIT_COND_CLASS ? 1 : 0) + c->depth * per_block + 4;
}

int adaln_bn(int R) {
  if (R <= 16) return 16;
  if (R <= 32) return 32;
  if (R <= 64) return 64;
  if (R <= 128) return 128;
  return 256;
}

}  // namespace

struct dit_handle {
  dit_config cfg;
  Geometry g;
  bool bf16 = false;
  int device = 0, num_sms = 148;
  std::string err;
  std::vector<void*> allocs;
  // weights
  float *pe_w = nullptr, *pe_wt = nullptr, *pe_b = nullptr, *t_w1 = nullptr, *t_b1 = nullptr, *t_w2 = nullptr,
        *t_b2 = nullptr;
  float* table = nullptr;
  void* ada_w = nullptr;
  float* ada_b = nullptr;
  std::vector<BlockW> blk;
  void* dec_w = nullptr;  // [dec_rows, d] bf16 or f32, rows >= P zero
  float* dec_b = nullptr;
  float *fln_s = nullptr, *fln_b = nullptr;  // final LayerNorm affine (gain - 1, bias) of the unmodulated designs
  float* ones = nullptr;                     // [d] of 1.0: the gate of the ungated designs
  uint8_t *u8 = nullptr, *g8 = nullptr;      // FP8 feed-forward operands [Mmax, d], [Mmax, mlp]
  float *su = nullptr, *sg = nullptr;        // their per-token scales [Mmax]
  uint8_t* o8 = nullptr;                     // FP8 attention output [Mmax, d] (the out-projection's operand)
  float* so = nullptr;                       // its per-token scales [Mmax]
  void* xkv_w = nullptr;                     // cross-attention key / value weights of all blocks [nkv, d]
  float *xkv_b = nullptr, *xkv = nullptr;    // their biases [nkv]; keys / values [2 Rmax, nkv] (f32)
  void* ctx = nullptr;                       // condition sequence [CTXalloc, d]: rows 2r, 2r+1 = e_t, e_y
  float *pos = nullptr, *rope = nullptr;
  // workspace
  float *E = nullptr, *hid = nullptr, *c = nullptr, *mod = nullptr, *h = nullptr, *z = nullptr;
  void *sc = nullptr, *u = nullptr, *q = nullptr, *k = nullptr, *v = nullptr, *o = nullptr, *gbuf = nullptr;
  int *status = nullptr, *probe_flag = nullptr;
  float *x_stage = nullptr, *t_stage = nullptr, *out_stage = nullptr;
  void* y_stage = nullptr;
  CUtensorMap tm_ada, tm_sc[5], tm_u, tm_o, tm_g, tm_dec, tm_xkv, tm_ctx[5];
  CUtensorMap tm_u8, tb_g8;  // FP8: LN output as fc1's A operand; fc1 output as fc2's B operand
  CUtensorMap tb_u8, tb_o8;  // FP8: LN output / attention output as the swapped GEMMs' B operand
  CUtensorMap tm_h_red;  // the residual stream as the TMA reduce-add target
  CUtensorMap tb_u, tb_o, tb_g;     // activations as the B operand of the swapped GEMMs (box 256 rows)
  AttnMaps attn_maps;
  int force_guidance = 0;
  int cfg_channels = 0;  // DIT_OPT_CFG_CHANNELS: guided output channels (0: all)
  int repeat_kind = -1;  // DIT_OPT_REPEAT_KIND: kernel kind launched twice per use (-1: none)
  int ksplit_short = 1;  // DIT_OPT_SPLIT_K: K slices of the short-K residual GEMMs (1: deterministic)
  int pair_gemm = 0;     // DIT_OPT_PAIR_GEMM: block GEMMs on SM pairs (tcgen05 cta_group::2)
  // CUDA-graph replay of the whole forward (DIT_OPT_USE_GRAPH): one cached executable graph,
  // valid for the exact pointers and parameters it was captured with
  struct GraphKey {
    const void *x, *t, *y;
    float* out;
    int B, R, depth, gch, rep;
    bool guided, pdl;
    float s;
    bool operator==(const GraphKey& o) const {
      return x == o.x && t == o.t && y == o.y && out == o.out && B == o.B && R == o.R && depth == o.depth &&
             gch == o.gch && rep == o.rep && guided == o.guided && pdl == o.pdl && s == o.s;
    }
  };
  cudaStream_t cap_stream = nullptr;
  cudaGraphExec_t gexec = nullptr;
  GraphKey gkey{}, gseen{};
  bool has_gseen = false;
  // dit_sample: per-step timestep table on the device and the cached graph of the loop
  float* t_sched = nullptr;
  size_t t_sched_cap = 0;
  std::vector<float> t_host;
  struct SampleKey {
    float* x = nullptr;
    const void* y = nullptr;
    const float* t_sched = nullptr;
    int B = 0, R = 0, kind = 0, steps = 0, gch = 0, rep = -1;
    bool guided = false, pdl = false;
    float s = 0.f;
    std::vector<float> levels;
    bool operator==(const SampleKey& o) const {
      return x == o.x && y == o.y && t_sched == o.t_sched && B == o.B && R == o.R && kind == o.kind && gch == o.gch &&
             rep == o.rep && steps == o.steps && guided == o.guided && pdl == o.pdl && s == o.s && levels == o.levels;
    }
  };
  cudaGraphExec_t sexec = nullptr;
  SampleKey skey, sseen;
  bool has_sseen = false;
  int use_graph = 0;
  // per-launch event timing (dit_profile_enable): every kind, or only prof_kind
  bool prof = false;
  int prof_kind = -1;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<std::pair<int, int>> prof_recs;  // (kind, index of the start event in ev_pool)

  template <typename T>
  T* alloc(size_t bytes, bool zero = true) {
    void* p = nullptr;
    if (bytes == 0) bytes = 16;
    if (cudaMalloc(&p, bytes) != cudaSuccess) return nullptr;
    allocs.push_back(p);
    if (zero) cudaMemset(p, 0, bytes);
    return static_cast<T*>(p);
  }
};

static dit_status fail(dit_handle* h, dit_status s, const std::string& m) {
  if (h) h->err = m;
  return s;
}

static dit_status cuda_fail(dit_handle* h, cudaError_t e, const char* where) {
  std::string m = std::string(where) + ": " + cudaGetErrorString(e);
  return fail(h, DIT_ERR_CUDA, m);
}

#define DIT_CK(h, call, where)                       \
  do {                                               \
    cudaError_t e_ = (call);                         \
    if (e_ != cudaSuccess) return cuda_fail(h, e_, where); \
  } while (0)

extern "C" {

int dit_weight_count(const dit_config* cfg) {
  std::string e;
  if (!validate(cfg, e)) return 0;
  return weight_count(cfg);
}

const char* dit_status_string(dit_status s) {
  switch (s) {
    case DIT_OK: return "DIT_OK";
    case DIT_ERR_INVALID_ARG: return "DIT_ERR_INVALID_ARG";
    case DIT_ERR_UNSUPPORTED: return "DIT_ERR_UNSUPPORTED";
    case DIT_ERR_OOM: return "DIT_ERR_OOM";
    case DIT_ERR_CUDA: return "DIT_ERR_CUDA";
    case DIT_ERR_DEVICE_TIMEOUT: return "DIT_ERR_DEVICE_TIMEOUT";
    case DIT_ERR_BAD_LABEL: return "DIT_ERR_BAD_LABEL";
    case DIT_ERR_NO_DEVICE: return "DIT_ERR_NO_DEVICE";
  }
  return "DIT_ERR_UNKNOWN";
}

const char* dit_last_error(const dit_handle* h) { return h ? h->err.c_str() : "null handle"; }

void dit_destroy(dit_handle* h) {
  if (h == nullptr) return;
  cudaDeviceSynchronize();
  if (h->gexec != nullptr) cudaGraphExecDestroy(h->gexec);
  if (h->sexec != nullptr) cudaGraphExecDestroy(h->sexec);
  if (h->t_sched != nullptr) cudaFree(h->t_sched);
  if (h->cap_stream != nullptr) cudaStreamDestroy(h->cap_stream);
  for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
  for (void* p : h->allocs) cudaFree(p);
  delete h;
}

// Upload one host float32 tensor to a float32 device buffer, or convert it to bf16
// through a float32 staging buffer.
static dit_status upload(dit_handle* H, const float* src, size_t n, void* dst, bool to_bf16, float* staging) {
  if (!to_bf16) {
    DIT_CK(H, cudaMemcpy(dst, src, n * 4, cudaMemcpyHostToDevice), "weight upload");
    return DIT_OK;
  }
  DIT_CK(H, cudaMemcpy(staging, src, n * 4, cudaMemcpyHostToDevice), "weight upload");
  DIT_CK(H, launch_f32_to_bf16(staging, static_cast<uint16_t*>(dst), n, 0), "bf16 convert");
  DIT_CK(H, cudaDeviceSynchronize(), "bf16 convert");
  return DIT_OK;
}

dit_status dit_create(const dit_config* cfg, const float* const* weights, int n_weights, dit_handle** out) {
  std::string err;
  if (out == nullptr) return DIT_ERR_INVALID_ARG;
  *out = nullptr;
  if (!validate(cfg, err)) return DIT_ERR_INVALID_ARG;
  if (weights == nullptr || n_weights != weight_count(cfg)) return DIT_ERR_INVALID_ARG;
  for (int i = 0; i < n_weights; ++i)
    if (weights[i] == nullptr) return DIT_ERR_INVALID_ARG;
  if (!supported(cfg, err)) return DIT_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIT_ERR_NO_DEVICE;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major != 10) return DIT_ERR_NO_DEVICE;

  dit_handle* H = new dit_handle();
  H->cfg = *cfg;
  H->g = geometry(cfg);
  H->bf16 = cfg->dtype == DIT_DTYPE_BF16;
  H->device = dev;
  H->num_sms = prop.multiProcessorCount;
  const Geometry& g = H->g;
  const int d = cfg->hidden, mlp = cfg->mlp_hidden, N = cfg->depth;
  const size_t es = H->bf16 ? 2 : 4;

#define ALLOC(ptr, T, bytes)                                      \
  do {                                                            \
    ptr = H->alloc<T>(bytes);                                     \
    if (ptr == nullptr) {                                         \
      dit_destroy(H);                                             \
      return DIT_ERR_OOM;                                         \
    }                                                             \
  } while (0)

  // ---------------- weights
  ALLOC(H->pe_w, float, (size_t)d * g.Kp * 4);
  ALLOC(H->pe_wt, float, (size_t)d * g.Kp * 4);
  ALLOC(H->pe_b, float, (size_t)d * 4);
  ALLOC(H->t_w1, float, (size_t)d * cfg->freq_dim * 4);
  ALLOC(H->t_b1, float, (size_t)d * 4);
  ALLOC(H->t_w2, float, (size_t)d * d * 4);
  ALLOC(H->t_b2, float, (size_t)d * 4);
  if (cfg->cond_kind == DIT_COND_CLASS) ALLOC(H->table, float, (size_t)(cfg->num_classes + 1) * d * 4);
  ALLOC(H->ada_w, void, (size_t)g.nmod * d * es);
  ALLOC(H->ada_b, float, (size_t)g.nmod * 4);
  const bool modulated = g.mpb > 0, cross = g.kind == DIT_BLOCK_CROSS_ATTN;
  ALLOC(H->ones, float, (size_t)d * 4);
  if (!modulated) {
    ALLOC(H->fln_s, float, (size_t)d * 4);
    ALLOC(H->fln_b, float, (size_t)d * 4);
  }
  if (cross) {
    ALLOC(H->xkv_w, void, (size_t)g.nkv * d * es);
    ALLOC(H->xkv_b, float, (size_t)g.nkv * 4);
  }
  H->blk.resize(N);
  for (int i = 0; i < N; ++i) {
    BlockW& b = H->blk[i];
    if (!modulated) {
      ALLOC(b.ln1_s, float, (size_t)d * 4);
      ALLOC(b.ln1_b, float, (size_t)d * 4);
      ALLOC(b.ln2_s, float, (size_t)d * 4);
      ALLOC(b.ln2_b, float, (size_t)d * 4);
    }
    if (cross) {
      ALLOC(b.xln_s, float, (size_t)d * 4);
      ALLOC(b.xln_b, float, (size_t)d * 4);
      ALLOC(b.xq_w, void, (size_t)d * d * es);
      ALLOC(b.xq_b, float, (size_t)d * 4);
      ALLOC(b.xo_w, void, (size_t)d * d * es);
      ALLOC(b.xo_b, float, (size_t)d * 4);
    }
    if (cfg->attn_fp8) {
      ALLOC(b.qkv_w8, uint8_t, (size_t)3 * d * d);
      ALLOC(b.qkv_s, float, (size_t)3 * d * 4);
      ALLOC(b.proj_w8, uint8_t, (size_t)d * d);
      ALLOC(b.proj_s, float, (size_t)d * 4);
    } else {
      ALLOC(b.qkv_w, void, (size_t)3 * d * d * es);
      ALLOC(b.proj_w, void, (size_t)d * d * es);
    }
    ALLOC(b.qkv_b, float, (size_t)3 * d * 4);
    ALLOC(b.proj_b, float, (size_t)d * 4);
    if (cfg->ffn_fp8) {
      ALLOC(b.fc1_w8, uint8_t, (size_t)mlp * d);
      ALLOC(b.fc1_s, float, (size_t)mlp * 4);
      ALLOC(b.fc2_w8, uint8_t, (size_t)d * mlp);
      ALLOC(b.fc2_s, float, (size_t)d * 4);
    } else {
      ALLOC(b.fc1_w, void, (size_t)mlp * d * es);
      ALLOC(b.fc2_w, void, (size_t)d * mlp * es);
    }
    ALLOC(b.fc1_b, float, (size_t)mlp * 4);
    ALLOC(b.fc2_b, float, (size_t)d * 4);
    if (cfg->qk_norm) {
      ALLOC(b.qn, float, (size_t)g.dh * 4);
      ALLOC(b.kn, float, (size_t)g.dh * 4);
    }
  }
  ALLOC(H->dec_w, void, (size_t)g.dec_rows * d * es);
  ALLOC(H->dec_b, float, (size_t)g.P * 4);
  if (cfg->pos_kind == DIT_POS_SINCOS2D) ALLOC(H->pos, float, (size_t)g.T * d * 4);
  else ALLOC(H->rope, float, (size_t)g.Ts * g.dh * 4);

  // ---------------- workspace
  const size_t R = g.Rmax, M = g.Mmax;
  ALLOC(H->E, float, R * cfg->freq_dim * 4);
  ALLOC(H->hid, float, R * d * 4);
  ALLOC(H->c, float, R * d * 4);
  ALLOC(H->sc, void, (size_t)g.RPalloc * d * es);
  ALLOC(H->mod, float, R * g.nmod * 4);
  if (cross) {
    ALLOC(H->ctx, void, (size_t)g.CTXalloc * d * es);
    ALLOC(H->xkv, float, 2 * R * g.nkv * 4);
  }
  ALLOC(H->h, float, M * d * 4);
  ALLOC(H->u, void, M * d * es);
  if (H->bf16) {
    const size_t qk = R * cfg->heads * (size_t)g.Tpad * g.DP * 2;
    ALLOC(H->q, void, qk);
    ALLOC(H->k, void, qk);
    ALLOC(H->v, void, qk);
  } else {
    const size_t qk = R * cfg->heads * (size_t)g.Ts * g.dh * 4;
    ALLOC(H->q, void, qk);
    ALLOC(H->k, void, qk);
    ALLOC(H->v, void, qk);
  }
  ALLOC(H->o, void, M * d * es);
  ALLOC(H->z, float, M * g.P * 4);
  if (cfg->ffn_fp8 || cfg->attn_fp8) {
    ALLOC(H->u8, uint8_t, M * d);
    ALLOC(H->su, float, M * 4);
    ALLOC(H->sg, float, M * 4);
  }
  if (cfg->attn_fp8) {
    ALLOC(H->o8, uint8_t, M * d);
    ALLOC(H->so, float, M * 4);
  }
  if (cfg->ffn_fp8) {
    ALLOC(H->g8, uint8_t, M * mlp);
    ALLOC(H->gbuf, void, 16);
  } else {
    ALLOC(H->gbuf, void, M * mlp * es);
  }
  ALLOC(H->status, int, 64);
  ALLOC(H->probe_flag, int, 64);
  const size_t xin = (size_t)cfg->max_batch * cfg->in_channels * cfg->frames * cfg->height * cfg->width;
  const size_t xout = (size_t)cfg->max_batch * g.Cout * cfg->frames * cfg->height * cfg->width;
  ALLOC(H->x_stage, float, xin * 4);
  ALLOC(H->t_stage, float, (size_t)cfg->max_batch * 4);
  ALLOC(H->y_stage, void, (size_t)cfg->max_batch * (cfg->cond_kind == DIT_COND_CLASS ? 4 : (size_t)d * 4));
  ALLOC(H->out_stage, float, xout * 4);

  // ---------------- upload
  size_t maxn = 0;
  {
    const size_t cand[] = {(size_t)3 * d * d, (size_t)mlp * d, (size_t)6 * d * d, (size_t)g.dec_rows * d};
    for (size_t v : cand) maxn = v > maxn ? v : maxn;
  }
  float* staging = nullptr;
  if (H->bf16) ALLOC(staging, float, maxn * 4);
  if ((cfg->ffn_fp8 || cfg->attn_fp8) && staging == nullptr) {
    dit_destroy(H);
    return DIT_ERR_INVALID_ARG;
  }
  int wi = 0;
  dit_status st = DIT_OK;
#define UP(dst, n, tobf)                                                 \
  do {                                                                   \
    st = upload(H, weights[wi++], (n), (dst), (tobf), staging);          \
    if (st != DIT_OK) {                                                  \
      dit_destroy(H);                                                    \
      return st;                                                         \
    }                                                                    \
  } while (0)
  {  // the patch weights also transposed, [Kp, d], for the embedding kernel's coalesced reads
    std::vector<float> wt((size_t)d * g.Kp);
    const float* w = weights[wi];
    for (int j = 0; j < d; ++j)
      for (int k = 0; k < g.Kp; ++k) wt[(size_t)k * d + j] = w[(size_t)j * g.Kp + k];
    if (cudaMemcpy(H->pe_wt, wt.data(), wt.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess) {
      dit_destroy(H);
      return DIT_ERR_CUDA;
    }
  }
  UP(H->pe_w, (size_t)d * g.Kp, false);
  UP(H->pe_b, (size_t)d, false);
  UP(H->t_w1, (size_t)d * cfg->freq_dim, false);
  UP(H->t_b1, (size_t)d, false);
  UP(H->t_w2, (size_t)d * d, false);
  UP(H->t_b2, (size_t)d, false);
  if (cfg->cond_kind == DIT_COND_CLASS) UP(H->table, (size_t)(cfg->num_classes + 1) * d, false);
  // a learned LayerNorm gain is stored as gain - 1 (the LN kernel applies (1 + scale))
#define UP_GAIN(dst)                                                        \
  do {                                                                      \
    std::vector<float> gm1(weights[wi], weights[wi] + d);                   \
    for (float& v : gm1) v -= 1.0f;                                         \
    ++wi;                                                                   \
    if (cudaMemcpy((dst), gm1.data(), (size_t)d * 4, cudaMemcpyHostToDevice) != cudaSuccess) { \
      dit_destroy(H);                                                       \
      return DIT_ERR_CUDA;                                                  \
    }                                                                       \
  } while (0)
  const int mpb = g.mpb;
  for (int i = 0; i < N; ++i) {
    BlockW& b = H->blk[i];
    if (modulated) {
      UP(static_cast<char*>(H->ada_w) + (size_t)i * mpb * d * d * es, (size_t)mpb * d * d, H->bf16);
      UP(H->ada_b + (size_t)i * mpb * d, (size_t)mpb * d, false);
    } else {
      UP_GAIN(b.ln1_s);
      UP(b.ln1_b, (size_t)d, false);
    }
    // E4M3 weights of the FP8 attention projections, quantised per output channel on the device
#define UP_E4M3(dst8, scale, rows)                                                                      \
  do {                                                                                                 \
    if (cudaMemcpy(staging, weights[wi++], (size_t)(rows) * d * 4, cudaMemcpyHostToDevice) != cudaSuccess || \
        launch_quantize_rows_e4m3(staging, (dst8), (scale), (rows), d, 0) != cudaSuccess ||              \
        cudaDeviceSynchronize() != cudaSuccess) {                                                      \
      dit_destroy(H);                                                                                  \
      return DIT_ERR_CUDA;                                                                             \
    }                                                                                                  \
  } while (0)
    if (cfg->attn_fp8)
      UP_E4M3(b.qkv_w8, b.qkv_s, 3 * d);
    else
      UP(b.qkv_w, (size_t)3 * d * d, H->bf16);
    UP(b.qkv_b, (size_t)3 * d, false);
    if (cfg->qk_norm) {
      UP(b.qn, (size_t)g.dh, false);
      UP(b.kn, (size_t)g.dh, false);
    }
    if (cfg->attn_fp8)
      UP_E4M3(b.proj_w8, b.proj_s, d);
    else
      UP(b.proj_w, (size_t)d * d, H->bf16);
    UP(b.proj_b, (size_t)d, false);
#undef UP_E4M3
    if (cross) {
      UP_GAIN(b.xln_s);
      UP(b.xln_b, (size_t)d, false);
      UP(b.xq_w, (size_t)d * d, H->bf16);
      UP(b.xq_b, (size_t)d, false);
      UP(static_cast<char*>(H->xkv_w) + (size_t)i * 2 * d * d * es, (size_t)2 * d * d, H->bf16);
      UP(H->xkv_b + (size_t)i * 2 * d, (size_t)2 * d, false);
      UP(b.xo_w, (size_t)d * d, H->bf16);
      UP(b.xo_b, (size_t)d, false);
    }
    if (!modulated) {
      UP_GAIN(b.ln2_s);
      UP(b.ln2_b, (size_t)d, false);
    }
    if (cfg->ffn_fp8) {
      // E4M3 weights, quantised per output channel on the device from the float32 values;
      // the hidden scale bound's constants from the host copy
      const float* w1 = weights[wi];
      double wmax = 0.0;
      for (int n = 0; n < mlp; ++n) {
        double ss = 0.0;
        for (int k = 0; k < d; ++k) ss += (double)w1[(size_t)n * d + k] * w1[(size_t)n * d + k];
        wmax = ss > wmax ? ss : wmax;
      }
      b.g_w = (float)std::sqrt(wmax);
      if (cudaMemcpy(staging, weights[wi++], (size_t)mlp * d * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
          launch_quantize_rows_e4m3(staging, b.fc1_w8, b.fc1_s, mlp, d, 0) != cudaSuccess ||
          cudaDeviceSynchronize() != cudaSuccess) {
        dit_destroy(H);
        return DIT_ERR_CUDA;
      }
      const float* b1 = weights[wi];
      float bmax = 0.f;
      for (int n = 0; n < mlp; ++n) bmax = fabsf(b1[n]) > bmax ? fabsf(b1[n]) : bmax;
      b.g_b = bmax;
      UP(b.fc1_b, (size_t)mlp, false);
      if (cudaMemcpy(staging, weights[wi++], (size_t)d * mlp * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
          launch_quantize_rows_e4m3(staging, b.fc2_w8, b.fc2_s, d, mlp, 0) != cudaSuccess ||
          cudaDeviceSynchronize() != cudaSuccess) {
        dit_destroy(H);
        return DIT_ERR_CUDA;
      }
      UP(b.fc2_b, (size_t)d, false);
    } else {
      UP(b.fc1_w, (size_t)mlp * d, H->bf16);
      UP(b.fc1_b, (size_t)mlp, false);
      UP(b.fc2_w, (size_t)d * mlp, H->bf16);
      UP(b.fc2_b, (size_t)d, false);
    }
  }
  if (modulated) {
    UP(static_cast<char*>(H->ada_w) + (size_t)N * mpb * d * d * es, (size_t)2 * d * d, H->bf16);
    UP(H->ada_b + (size_t)N * mpb * d, (size_t)2 * d, false);
  } else {
    UP_GAIN(H->fln_s);
    UP(H->fln_b, (size_t)d, false);
  }
#undef UP_GAIN
  {
    std::vector<float> one((size_t)d, 1.0f);
    if (cudaMemcpy(H->ones, one.data(), (size_t)d * 4, cudaMemcpyHostToDevice) != cudaSuccess) {
      dit_destroy(H);
      return DIT_ERR_CUDA;
    }
  }
  UP(H->dec_w, (size_t)g.P * d, H->bf16);
  UP(H->dec_b, (size_t)g.P, false);
#undef UP
#undef ALLOC

  if (launch_pos_tables(H->pos, H->rope, g.gf, g.gh, g.gw, d, g.dh, g.Tc, 0) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    dit_destroy(H);
    return DIT_ERR_CUDA;
  }

  // ---------------- tensor maps (bf16 path)
  if (H->bf16) {
    bool ok = g.nmod == 0 || make_tmap_bf16_kmajor(&H->tm_ada, H->ada_w, g.nmod, d, 128);
    const int bns[5] = {16, 32, 64, 128, 256};
    for (int i = 0; i < 5; ++i) ok = ok && make_tmap_bf16_kmajor(&H->tm_sc[i], H->sc, g.RPalloc, d, bns[i]);
    if (cross) {
      ok = ok && make_tmap_bf16_kmajor(&H->tm_xkv, H->xkv_w, g.nkv, d, 128);
      for (int i = 0; i < 5; ++i) ok = ok && make_tmap_bf16_kmajor(&H->tm_ctx[i], H->ctx, g.CTXalloc, d, bns[i]);
    }
    ok = ok && make_tmap_bf16_kmajor(&H->tm_u, H->u, g.Mmax, d, 128);
    ok = ok && make_tmap_bf16_kmajor(&H->tm_o, H->o, g.Mmax, d, 128);
    if (cfg->ffn_fp8 || cfg->attn_fp8)
      ok = ok && make_tmap_e4m3_kmajor(&H->tm_u8, H->u8, g.Mmax, d, 128) &&
           make_tmap_e4m3_kmajor(&H->tb_u8, H->u8, g.Mmax, d, 256);
    if (cfg->attn_fp8) ok = ok && make_tmap_e4m3_kmajor(&H->tb_o8, H->o8, g.Mmax, d, 256);
    if (cfg->ffn_fp8) {
      ok = ok && make_tmap_e4m3_kmajor(&H->tb_g8, H->g8, g.Mmax, mlp, 256);
    } else {
      ok = ok && make_tmap_bf16_kmajor(&H->tm_g, H->gbuf, g.Mmax, mlp, 128) &&
           make_tmap_bf16_kmajor(&H->tb_g, H->gbuf, g.Mmax, mlp, 256);
    }
    ok = ok && make_tmap_bf16_kmajor(&H->tm_dec, H->dec_w, g.dec_rows, d, g.bn_dec);
    ok = ok && make_tmap_f32(&H->tm_h_red, H->h, g.Mmax, d, 32, 16, 128);
    ok = ok && make_tmap_bf16_kmajor(&H->tb_u, H->u, g.Mmax, d, 256);
    ok = ok && make_tmap_bf16_kmajor(&H->tb_o, H->o, g.Mmax, d, 256);
    ok = ok && make_attention_maps(&H->attn_maps, H->q, H->k, H->v, H->o, g.Rmax, cfg->heads, g.Ts, g.Tpad, g.dh, g.DP, d);
    for (int i = 0; i < N && ok; ++i) {
      BlockW& b = H->blk[i];
      if (cfg->attn_fp8)
        ok = make_tmap_e4m3_kmajor(&b.tm_qkv8, b.qkv_w8, 3 * d, d, g.headwise ? g.bn_qkv : 128) &&
             make_tmap_e4m3_kmajor(&b.ta_qkv8, b.qkv_w8, 3 * d, d, 128) &&
             make_tmap_e4m3_kmajor(&b.ta_proj8, b.proj_w8, d, d, 128);
      else
        ok = make_tmap_bf16_kmajor(&b.tm_qkv, b.qkv_w, 3 * d, d, g.headwise ? g.bn_qkv : 128) &&
             make_tmap_bf16_kmajor(&b.ta_qkv, b.qkv_w, 3 * d, d, 128) &&
             make_tmap_bf16_kmajor(&b.ta_proj, b.proj_w, d, d, 128);
      if (cfg->ffn_fp8)
        ok = ok && make_tmap_e4m3_kmajor(&b.tm_fc1_8, b.fc1_w8, mlp, d, g.bn_fc1) &&
             make_tmap_e4m3_kmajor(&b.ta_fc2_8, b.fc2_w8, d, mlp, 128);
      else
        ok = ok && make_tmap_bf16_kmajor(&b.tm_fc1, b.fc1_w, mlp, d, g.bn_fc1) &&
             make_tmap_bf16_kmajor(&b.tm_fc1_h, b.fc1_w, mlp, d, 128) &&
             make_tmap_bf16_kmajor(&b.ta_fc2, b.fc2_w, d, mlp, 128);
      if (cross)
        ok = ok && make_tmap_bf16_kmajor(&b.tm_xq, b.xq_w, d, d, 2 * g.dh) &&
             make_tmap_bf16_kmajor(&b.ta_xo, b.xo_w, d, d, 128);
    }
    if (!ok) {
      dit_destroy(H);
      return DIT_ERR_CUDA;
    }
  }
  *out = H;
  return DIT_OK;
}

int dit_forward_launch_count(const dit_handle* H, int B, float cfg_scale) {
  if (H == nullptr) return 0;
  (void)B;
  (void)cfg_scale;
  const Geometry& g = H->g;
  int per_block = 7 + ((!H->bf16 && (H->cfg.qk_norm || H->cfg.pos_kind == DIT_POS_ROPE3D)) ? 1 : 0) +
                  (H->cfg.attn_fp8 ? 1 : 0);  // the attention output's E4M3 quantisation
  if (g.kind == DIT_BLOCK_CROSS_ATTN) per_block += H->bf16 ? 3 : 4;
  const int front = 3 + (g.nmod > 0 ? 1 : 0) + (g.nkv > 0 ? 1 : 0) + 1;  // condition, projections, embedding
  return front + H->cfg.depth * per_block + 1 + 2;
}

}  // extern "C"

// --------------------------------------------------------------------------- forward
namespace {

struct RunPlan {
  int B, R, M;
  bool guided;
  float s;
};

dit_status check_run(dit_handle* H, const void* x, const void* t, const void* y, int B, float s, RunPlan& p) {
  if (H == nullptr) return DIT_ERR_INVALID_ARG;
  if (x == nullptr || t == nullptr || y == nullptr) return fail(H, DIT_ERR_INVALID_ARG, "null input pointer");
  if (B < 1 || B > H->cfg.max_batch) return fail(H, DIT_ERR_INVALID_ARG, "batch outside [1, max_batch]");
  if (!isfinite(s)) return fail(H, DIT_ERR_INVALID_ARG, "cfg_scale must be finite");
  p.B = B;
  p.guided = H->cfg.cond_kind == DIT_COND_CLASS && (s != 1.0f || H->force_guidance);
  p.R = p.guided ? 2 * B : B;
  p.M = p.R * H->g.Ts;
  p.s = s;
  return DIT_OK;
}

bool prof_on(const dit_handle* H, int kind) { return H->prof && (H->prof_kind < 0 || H->prof_kind == kind); }

void prof_begin(dit_handle* H, int kind, cudaStream_t st) {
  if (!prof_on(H, kind)) return;
  const size_t i = H->prof_recs.size() * 2;
  while (H->ev_pool.size() < i + 2) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    H->ev_pool.push_back(e);
  }
  H->prof_recs.push_back({kind, static_cast<int>(i)});
  cudaEventRecord(H->ev_pool[i], st);
}

void prof_end(dit_handle* H, int kind, cudaStream_t st) {
  if (!prof_on(H, kind) || H->prof_recs.empty()) return;
  cudaEventRecord(H->ev_pool[H->prof_recs.back().second + 1], st);
}

// Launches `call` once (twice when DIT_OPT_REPEAT_KIND names its kind: a timing
// diagnostic, the step time grows by the kind's in-pipeline cost).
#define DIT_LAUNCH(H, kind, st, call, where)           \
  do {                                                \
    prof_begin(H, kind, st);                          \
    DIT_CK(H, call, where);                           \
    if (H->repeat_kind == (kind)) DIT_CK(H, call, where); \
    prof_end(H, kind, st);                            \
  } while (0)

dit_status run_condition(dit_handle* H, const float* t, const void* y, const RunPlan& p, cudaStream_t st) {
  const dit_config& c = H->cfg;
  const Geometry& g = H->g;
  CondArgs a;
  a.t = t;
  a.y = y;
  a.B = p.B;
  a.R = p.R;
  a.d = c.hidden;
  a.freq = c.freq_dim;
  a.cond_kind = c.cond_kind;
  a.num_classes = c.num_classes;
  a.guided = p.guided;
  a.t_scale = c.t_scale;
  a.w1 = H->t_w1;
  a.b1 = H->t_b1;
  a.w2 = H->t_w2;
  a.b2 = H->t_b2;
  a.table = H->table;
  a.E = H->E;
  a.hid = H->hid;
  a.c = H->c;
  a.sc = g.mpb > 0 ? H->sc : nullptr;  // SiLU(c) feeds the modulation GEMM
  a.sc_bf16 = H->bf16;
  a.status = H->status;
  if (g.kind == DIT_BLOCK_IN_CONTEXT) {  // e_t, e_y as the first two tokens of every row
    a.tok_h = H->h;
    a.tok_ld = (size_t)g.Ts * c.hidden;
  } else if (g.kind == DIT_BLOCK_CROSS_ATTN) {  // e_t, e_y as the condition sequence
    a.ctx = H->ctx;
    a.ctx_bf16 = H->bf16;
  }
  DIT_LAUNCH(H, DIT_KERNEL_COND, st, launch_condition(a, st), "condition");
  return DIT_OK;
}

// Row-independent (scale, shift) or per-row modulation vectors of one normalisation.
struct Norm {
  const float *shift, *scale;
  int ld;
};

// Runs the forward through `stop_after` blocks (depth => the whole network, with
// the final layer when out != nullptr).
dit_status run_forward(dit_handle* H, const float* x, const float* t, const void* y, const RunPlan& p, int stop_after,
                       float* out, cudaStream_t st) {
  const dit_config& c = H->cfg;
  const Geometry& g = H->g;
  const int d = c.hidden, mlp = c.mlp_hidden, Ts = g.Ts;
  dit_status s = run_condition(H, t, y, p, st);
  if (s != DIT_OK) return s;

  // modulation vectors of every block and the final layer: mod[r, nmod] (modulated designs)
  if (g.nmod > 0) {
    EpiArgs ea = {};
    ea.M = g.nmod;
    ea.N = p.R;
    ea.bias = H->ada_b;
    ea.out = H->mod;
    ea.ldo = g.nmod;
    ea.status = H->status;
    if (H->bf16) {
      const int bn = adaln_bn(p.R);
      const int idx = bn == 16 ? 0 : bn == 32 ? 1 : bn == 64 ? 2 : bn == 128 ? 3 : 4;
      DIT_LAUNCH(H, DIT_KERNEL_ADALN, st, launch_gemm_tc(EPI_ADALN, bn, &H->tm_ada, &H->tm_sc[idx], d, ea, H->num_sms, st), "adaLN gemm");
    } else {
      DIT_LAUNCH(H, DIT_KERNEL_ADALN, st, launch_gemm_simt(EPI_ADALN, static_cast<const float*>(H->ada_w), static_cast<const float*>(H->sc),
                                 g.nmod, p.R, d, ea, st),
             "adaLN gemm");
    }
  }
  // cross-attention keys and values of every block from the two condition tokens:
  // xkv[2r + s, blk * 2d + (0: k | d: v)]
  if (g.nkv > 0) {
    EpiArgs ea = {};
    ea.M = g.nkv;
    ea.N = 2 * p.R;
    ea.bias = H->xkv_b;
    ea.out = H->xkv;
    ea.ldo = g.nkv;
    ea.status = H->status;
    if (H->bf16) {
      const int bn = adaln_bn(2 * p.R);
      const int idx = bn == 16 ? 0 : bn == 32 ? 1 : bn == 64 ? 2 : bn == 128 ? 3 : 4;
      DIT_LAUNCH(H, DIT_KERNEL_ADALN, st, launch_gemm_tc(EPI_ADALN, bn, &H->tm_xkv, &H->tm_ctx[idx], d, ea, H->num_sms, st),
                 "condition key / value gemm");
    } else {
      DIT_LAUNCH(H, DIT_KERNEL_ADALN, st,
                 launch_gemm_simt(EPI_ADALN, static_cast<const float*>(H->xkv_w), static_cast<const float*>(H->ctx),
                                  g.nkv, 2 * p.R, d, ea, st),
                 "condition key / value gemm");
    }
  }
  {
    PatchArgs a;
    a.x = x;
    a.w = H->pe_w;
    a.wt = H->pe_wt;
    a.b = H->pe_b;
    a.pos = H->pos;
    a.h = H->h;
    a.B = p.B;
    a.R = p.R;
    a.C = c.in_channels;
    a.F = c.frames;
    a.H = c.height;
    a.W = c.width;
    a.pt = c.patch_t;
    a.ph = c.patch_h;
    a.pw = c.patch_w;
    a.d = d;
    a.Trow = Ts;
    a.tok0 = g.Tc;
    DIT_LAUNCH(H, DIT_KERNEL_PATCH, st, launch_patch_embed(a, st), "patch embed");
  }
  auto run_ln = [&](const Norm& n, const char* where) -> dit_status {
    LnArgs ln;
    ln.h = H->h;
    ln.u = H->u;
    ln.u_bf16 = H->bf16;
    ln.ld_mod = n.ld;
    ln.M = p.M;
    ln.T = Ts;
    ln.d = d;
    ln.shift = n.shift;
    ln.scale = n.scale;
    DIT_LAUNCH(H, DIT_KERNEL_LN, st, launch_ln_modulate(ln, st), where);
    return DIT_OK;
  };
  // gated residual update h += gate[row] * (A W^T + b) on the tensor cores (swapped operands)
  // or the SIMT GEMM
  // tb: the activations as the B operand (256-row box); tb_half: the same with a 128-row box
  // for the SM-pair GEMM (nullptr: no pair variant)
  auto run_resid = [&](int kind, const CUtensorMap* ta, const CUtensorMap* tb, const CUtensorMap* tb_half,
                       const void* A, const void* W, int K, const float* bias, const float* gate, int ld_gate,
                       const char* where) -> dit_status {
    EpiArgs pa = {};
    pa.M = p.M;
    pa.N = d;
    pa.bias = bias;
    pa.h = H->h;
    pa.ldh = d;
    pa.gate = gate;
    pa.ld_gate = ld_gate;
    pa.T = Ts;
    pa.status = H->status;
    if (H->bf16) {
      EpiArgs pt = pa;  // swapped: rows = d output features, columns = tokens
      pt.M = d;
      pt.N = p.M;
      // short K (the d-wide projections): two K slices double the work units per SM, so
      // the pipeline fill and the last epilogue are no longer exposed
      pt.ksplit = K <= 2048 ? H->ksplit_short : 1;
      if (H->pair_gemm && tb_half != nullptr)
        DIT_LAUNCH(H, kind, st, launch_gemm_tc2(EPI_RESID_T, 256, ta, tb_half, K, pt, H->num_sms, st, &H->tm_h_red),
                   where);
      else
        DIT_LAUNCH(H, kind, st, launch_gemm_tc(EPI_RESID_T, 256, ta, tb, K, pt, H->num_sms, st, &H->tm_h_red), where);
    } else {
      DIT_LAUNCH(H, kind, st,
                 launch_gemm_simt(EPI_RESID, static_cast<const float*>(A), static_cast<const float*>(W), p.M, d, K, pa, st),
                 where);
    }
    return DIT_OK;
  };
#define DIT_TRY(call)               \
  do {                              \
    const dit_status s_ = (call);   \
    if (s_ != DIT_OK) return s_;    \
  } while (0)

  const bool modulated = g.mpb > 0;
  const int nblk = stop_after < c.depth ? stop_after : c.depth;
  for (int i = 0; i < nblk; ++i) {
    BlockW& b = H->blk[i];
    const float* mb = modulated ? H->mod + (size_t)i * g.mpb * d : nullptr;
    Norm n1, n2;
    const float *gate1 = H->ones, *gate2 = H->ones;
    int ld_gate = 0;
    if (g.kind == DIT_BLOCK_ADALN_ZERO) {  // (shift1, scale1, gate1, shift2, scale2, gate2)
      n1 = {mb, mb + d, g.nmod};
      n2 = {mb + 3 * d, mb + 4 * d, g.nmod};
      gate1 = mb + 2 * d;
      gate2 = mb + 5 * d;
      ld_gate = g.nmod;
    } else if (g.kind == DIT_BLOCK_ADALN) {  // (shift1, scale1, shift2, scale2), no gates
      n1 = {mb, mb + d, g.nmod};
      n2 = {mb + 2 * d, mb + 3 * d, g.nmod};
    } else {  // learned LayerNorm affines, the same for every row
      n1 = {b.ln1_b, b.ln1_s, 0};
      n2 = {b.ln2_b, b.ln2_s, 0};
    }
    if (c.attn_fp8) {  // LN1 straight to E4M3 with per-token scales (the in-projection's operand)
      LnArgs ln;
      ln.h = H->h;
      ln.u = H->u;
      ln.u_bf16 = 1;
      ln.u8 = H->u8;
      ln.su = H->su;
      ln.sg = H->sg;  // written, unused: no GELU follows
      ln.g_w = 0.f;
      ln.g_b = 0.f;
      ln.ld_mod = n1.ld;
      ln.M = p.M;
      ln.T = Ts;
      ln.d = d;
      ln.shift = n1.shift;
      ln.scale = n1.scale;
      DIT_LAUNCH(H, DIT_KERNEL_LN, st, launch_ln_modulate(ln, st), "ln1 (fp8)");
    } else {
      DIT_TRY(run_ln(n1, "ln1"));
    }

    EpiArgs qa = {};
    qa.M = p.M;
    qa.N = 3 * d;
    qa.bias = b.qkv_b;
    qa.q = H->q;
    qa.k = H->k;
    qa.v = H->v;
    qa.d = d;
    qa.H = c.heads;
    qa.dh = g.dh;
    qa.DP = g.DP;
    qa.Tpad = g.Tpad;
    qa.T = Ts;
    qa.qn = b.qn;
    qa.kn = b.kn;
    qa.rope = H->rope;
    qa.status = H->status;
    AttnArgs aa;
    aa.q = H->q;
    aa.k = H->k;
    aa.v = H->v;
    aa.o = H->o;
    aa.R = p.R;
    aa.H = c.heads;
    aa.T = Ts;
    aa.dh = g.dh;
    aa.DP = g.DP;
    aa.Tpad = g.Tpad;
    aa.d = d;
    aa.bf16 = H->bf16;

    if (H->bf16 && c.attn_fp8) {  // E4M3 in-projection (kind::f8f6f4), scales applied in the epilogue
      if (g.headwise) {
        EpiArgs q8 = qa;
        q8.sa = H->su;
        q8.sb = b.qkv_s;
        DIT_LAUNCH(H, DIT_KERNEL_QKV, st,
                   launch_gemm_tc(EPI_QKV_HEAD8, g.bn_qkv, &H->tm_u8, &b.tm_qkv8, d, q8, H->num_sms, st),
                   "qkv gemm (fp8)");
      } else {
        EpiArgs q8 = qa;  // swapped: rows = 3d output features, columns = tokens
        q8.M = 3 * d;
        q8.N = p.M;
        q8.sa = b.qkv_s;
        q8.sb = H->su;
        DIT_LAUNCH(H, DIT_KERNEL_QKV, st,
                   launch_gemm_tc(EPI_QKV_T8, 256, &b.ta_qkv8, &H->tb_u8, d, q8, H->num_sms, st), "qkv gemm (fp8)");
      }
      DIT_LAUNCH(H, DIT_KERNEL_ATTN, st, launch_attention_tc(aa, H->attn_maps, H->status, st), "attention");
    } else if (H->bf16) {
      if (g.headwise) {
        DIT_LAUNCH(H, DIT_KERNEL_QKV, st,
                   launch_gemm_tc(EPI_QKV_HEAD, g.bn_qkv, &H->tm_u, &b.tm_qkv, d, qa, H->num_sms, st), "qkv gemm");
      } else {
        EpiArgs qt = qa;  // swapped: rows = 3d output features, columns = tokens
        qt.M = 3 * d;
        qt.N = p.M;
        if (H->pair_gemm)
          DIT_LAUNCH(H, DIT_KERNEL_QKV, st, launch_gemm_tc2(EPI_QKV_T, 256, &b.ta_qkv, &H->tm_u, d, qt, H->num_sms, st),
                     "qkv gemm");
        else
          DIT_LAUNCH(H, DIT_KERNEL_QKV, st, launch_gemm_tc(EPI_QKV_T, 256, &b.ta_qkv, &H->tb_u, d, qt, H->num_sms, st),
                     "qkv gemm");
      }
      DIT_LAUNCH(H, DIT_KERNEL_ATTN, st, launch_attention_tc(aa, H->attn_maps, H->status, st), "attention");
    } else {
      DIT_LAUNCH(H, DIT_KERNEL_QKV, st, launch_gemm_simt(EPI_QKV, static_cast<const float*>(H->u), static_cast<const float*>(b.qkv_w), p.M,
                                 3 * d, d, qa, st),
             "qkv gemm");
      if (c.qk_norm || c.pos_kind == DIT_POS_ROPE3D) {
        QkNormArgs qn;
        qn.q = static_cast<float*>(H->q);
        qn.k = static_cast<float*>(H->k);
        qn.qn = b.qn;
        qn.kn = b.kn;
        qn.rope = H->rope;
        qn.RH = p.R * c.heads;
        qn.T = Ts;
        qn.dh = g.dh;
        DIT_LAUNCH(H, DIT_KERNEL_QKV, st, launch_qknorm_rope_f32(qn, st), "qk norm");
      }
      DIT_LAUNCH(H, DIT_KERNEL_ATTN, st, launch_attention_simt(aa, st), "attention");
    }
    if (c.attn_fp8) {  // the heads' output to E4M3 per token, then the E4M3 out-projection
      DIT_LAUNCH(H, DIT_KERNEL_PROJ, st,
                 launch_quantize_rows_bf16_e4m3(static_cast<const uint16_t*>(H->o), H->o8, H->so, p.M, d, st),
                 "attention output to e4m3");
      EpiArgs pt = {};
      pt.M = d;
      pt.N = p.M;
      pt.bias = b.proj_b;
      pt.h = H->h;
      pt.ldh = d;
      pt.gate = gate1;
      pt.ld_gate = ld_gate;
      pt.T = Ts;
      pt.sa = b.proj_s;
      pt.sb = H->so;
      pt.status = H->status;
      DIT_LAUNCH(H, DIT_KERNEL_PROJ, st,
                 launch_gemm_tc(EPI_RESID_T8, 256, &b.ta_proj8, &H->tb_o8, d, pt, H->num_sms, st, &H->tm_h_red),
                 "proj gemm (fp8)");
    } else {
      DIT_TRY(run_resid(DIT_KERNEL_PROJ, &b.ta_proj, &H->tb_o, &H->tm_o, H->o, b.proj_w, d, b.proj_b, gate1, ld_gate,
                        "proj gemm"));
    }

    if (g.kind == DIT_BLOCK_CROSS_ATTN) {  // h += CrossAttn(LNx(h), [e_t, e_y])
      DIT_TRY(run_ln(Norm{b.xln_b, b.xln_s, 0}, "cross-attention ln"));
      const float* xkv = H->xkv + (size_t)i * 2 * d;
      if (H->bf16) {
        EpiArgs xa = {};
        xa.M = p.M;
        xa.N = d;
        xa.bias = b.xq_b;
        xa.xkv = xkv;
        xa.ld_xkv = g.nkv;
        xa.xo = H->o;
        xa.d = d;
        xa.T = Ts;
        xa.status = H->status;
        DIT_LAUNCH(H, DIT_KERNEL_ATTN, st, launch_gemm_tc(EPI_XATTN, 2 * g.dh, &H->tm_u, &b.tm_xq, d, xa, H->num_sms, st),
                   "cross-attention query gemm");
      } else {
        EpiArgs xa = {};
        xa.M = p.M;
        xa.N = d;
        xa.bias = b.xq_b;
        xa.out = H->q;  // [M, d] float32 queries (the q buffer is free until the next block)
        xa.ldo = d;
        xa.status = H->status;
        DIT_LAUNCH(H, DIT_KERNEL_ATTN, st,
                   launch_gemm_simt(EPI_F32, static_cast<const float*>(H->u), static_cast<const float*>(b.xq_w), p.M, d,
                                    d, xa, st),
                   "cross-attention query gemm");
        XAttnArgs xk;
        xk.q = static_cast<const float*>(H->q);
        xk.xkv = xkv;
        xk.ld_xkv = g.nkv;
        xk.o = static_cast<float*>(H->o);
        xk.M = p.M;
        xk.T = Ts;
        xk.d = d;
        xk.H = c.heads;
        xk.dh = g.dh;
        DIT_LAUNCH(H, DIT_KERNEL_ATTN, st, launch_xattn_f32(xk, st), "cross-attention");
      }
      DIT_TRY(run_resid(DIT_KERNEL_PROJ, &b.ta_xo, &H->tb_o, &H->tm_o, H->o, b.xo_w, d, b.xo_b, H->ones, 0,
                        "cross-attention output gemm"));
    }

    if (c.ffn_fp8) {  // feed-forward with E4M3 operands on the tensor cores (kind::f8f6f4)
      LnArgs ln;
      ln.h = H->h;
      ln.u = H->u;
      ln.u_bf16 = 1;
      ln.u8 = H->u8;
      ln.su = H->su;
      ln.sg = H->sg;
      ln.g_w = b.g_w;
      ln.g_b = b.g_b;
      ln.ld_mod = n2.ld;
      ln.M = p.M;
      ln.T = Ts;
      ln.d = d;
      ln.shift = n2.shift;
      ln.scale = n2.scale;
      DIT_LAUNCH(H, DIT_KERNEL_LN, st, launch_ln_modulate(ln, st), "ln2 (fp8)");
      EpiArgs f1 = {};
      f1.M = p.M;
      f1.N = mlp;
      f1.bias = b.fc1_b;
      f1.out = H->g8;
      f1.ldo = mlp;
      f1.sa = H->su;
      f1.sb = b.fc1_s;
      f1.sg = H->sg;
      f1.status = H->status;
      DIT_LAUNCH(H, DIT_KERNEL_FC1, st, launch_gemm_tc(EPI_GELU8, 256, &H->tm_u8, &b.tm_fc1_8, d, f1, H->num_sms, st),
                 "fc1 gemm (fp8)");
      EpiArgs f2 = {};
      f2.M = d;
      f2.N = p.M;
      f2.bias = b.fc2_b;
      f2.h = H->h;
      f2.ldh = d;
      f2.gate = gate2;
      f2.ld_gate = ld_gate;
      f2.T = Ts;
      f2.sa = b.fc2_s;
      f2.sb = H->sg;
      f2.status = H->status;
      DIT_LAUNCH(H, DIT_KERNEL_FC2, st,
                 launch_gemm_tc(EPI_RESID_T8, 256, &b.ta_fc2_8, &H->tb_g8, mlp, f2, H->num_sms, st, &H->tm_h_red),
                 "fc2 gemm (fp8)");
      continue;
    }
    DIT_TRY(run_ln(n2, "ln2"));
    EpiArgs f1 = {};
    f1.M = p.M;
    f1.N = mlp;
    f1.bias = b.fc1_b;
    f1.out = H->gbuf;
    f1.ldo = mlp;
    f1.status = H->status;
    if (H->bf16) {
      if (H->pair_gemm)
        DIT_LAUNCH(H, DIT_KERNEL_FC1, st,
                   launch_gemm_tc2(EPI_GELU, 256, &H->tm_u, &b.tm_fc1_h, d, f1, H->num_sms, st),
                   "fc1 gemm");
      else
        DIT_LAUNCH(H, DIT_KERNEL_FC1, st,
                   launch_gemm_tc(EPI_GELU, g.bn_fc1, &H->tm_u, &b.tm_fc1, d, f1, H->num_sms, st),
                   "fc1 gemm");
    } else {
      DIT_LAUNCH(H, DIT_KERNEL_FC1, st, launch_gemm_simt(EPI_GELU, static_cast<const float*>(H->u), static_cast<const float*>(b.fc1_w), p.M,
                                 mlp, d, f1, st),
             "fc1 gemm");
    }
    DIT_TRY(run_resid(DIT_KERNEL_FC2, &b.ta_fc2, &H->tb_g, &H->tm_g, H->gbuf, b.fc2_w, mlp, b.fc2_b, gate2, ld_gate,
                      "fc2 gemm"));
  }
  if (out == nullptr) return DIT_OK;

  // final layer: modulated (adaLN designs) or learned-affine LayerNorm
  if (modulated) {
    const float* fm = H->mod + (size_t)c.depth * g.mpb * d;
    DIT_TRY(run_ln(Norm{fm, fm + d, g.nmod}, "final ln"));
  } else {
    DIT_TRY(run_ln(Norm{H->fln_b, H->fln_s, 0}, "final ln"));
  }
#undef DIT_TRY
  // linear decoder z = u W_dec^T + b_dec [M, P] (tensor cores on the bf16 path), then the
  // guidance combine and unpatchify (condition tokens are skipped)
  EpiArgs de = {};
  de.M = p.M;
  de.N = g.P;
  de.bias = H->dec_b;
  de.out = H->z;
  de.ldo = g.P;
  de.status = H->status;
  if (H->bf16) {
    DIT_LAUNCH(H, DIT_KERNEL_DECODE, st, launch_gemm_tc(EPI_F32, g.bn_dec, &H->tm_u, &H->tm_dec, d, de, H->num_sms, st),
               "decoder gemm");
  } else {
    DIT_LAUNCH(H, DIT_KERNEL_DECODE, st,
               launch_gemm_simt(EPI_F32, static_cast<const float*>(H->u), static_cast<const float*>(H->dec_w), p.M, g.P,
                                d, de, st),
               "decoder gemm");
  }
  UnpatchArgs ua;
  ua.z = H->z;
  ua.out = out;
  ua.B = p.B;
  ua.T = g.T;
  ua.P = g.P;
  ua.Cout = g.Cout;
  ua.F = c.frames;
  ua.H = c.height;
  ua.W = c.width;
  ua.pt = c.patch_t;
  ua.ph = c.patch_h;
  ua.pw = c.patch_w;
  ua.guided = p.guided;
  ua.s = p.s;
  ua.gch = H->cfg_channels;
  ua.Trow = Ts;
  ua.tok0 = g.Tc;
  DIT_LAUNCH(H, DIT_KERNEL_DECODE, st, launch_cfg_unpatchify(ua, H->num_sms, st), "guidance + unpatchify");
  return DIT_OK;
}

// The forward through a cached CUDA graph when DIT_OPT_USE_GRAPH is on.  A new set of
// pointers / parameters runs directly the first time it is seen (which also performs the
// kernels' one-time attribute set-up), is captured on a private stream the second time,
// and replays as one graph launch on the caller's stream from then on.  A capture that
// fails turns the option off and runs directly.
dit_status run_forward_cached(dit_handle* H, const float* x, const float* t, const void* y, const RunPlan& p,
                              float* out, cudaStream_t st) {
  const int depth = H->cfg.depth;
  if (!H->use_graph || H->prof) return run_forward(H, x, t, y, p, depth, out, st);
  dit_handle::GraphKey k{x, t, y, out, p.B, p.R, depth, H->cfg_channels, H->repeat_kind, p.guided, g_pdl, p.s};
  if (H->gexec != nullptr && k == H->gkey) {
    DIT_CK(H, cudaGraphLaunch(H->gexec, st), "graph launch");
    return DIT_OK;
  }
  if (!(H->has_gseen && k == H->gseen)) {
    H->gseen = k;
    H->has_gseen = true;
    return run_forward(H, x, t, y, p, depth, out, st);
  }
  if (H->cap_stream == nullptr) DIT_CK(H, cudaStreamCreateWithFlags(&H->cap_stream, cudaStreamNonBlocking), "capture stream");
  DIT_CK(H, cudaStreamBeginCapture(H->cap_stream, cudaStreamCaptureModeThreadLocal), "begin capture");
  const dit_status s = run_forward(H, x, t, y, p, depth, out, H->cap_stream);
  cudaGraph_t graph = nullptr;
  cudaError_t e = cudaStreamEndCapture(H->cap_stream, &graph);
  cudaGraphExec_t ex = nullptr;
  if (s == DIT_OK && e == cudaSuccess) e = cudaGraphInstantiate(&ex, graph, 0);
  if (graph != nullptr) cudaGraphDestroy(graph);
  if (s != DIT_OK || e != cudaSuccess || ex == nullptr) {
    cudaGetLastError();
    H->use_graph = 0;
    if (s != DIT_OK) return s;
    return run_forward(H, x, t, y, p, depth, out, st);
  }
  if (H->gexec != nullptr) cudaGraphExecDestroy(H->gexec);
  H->gexec = ex;
  H->gkey = k;
  DIT_CK(H, cudaGraphLaunch(H->gexec, st), "graph launch");
  return DIT_OK;
}

// One sampler update (the coefficients of x_next = c0 x + c1 pred formed in double).
dit_status enqueue_sampler_step(dit_handle* H, int kind, const float* x, const float* pred, int B, float a, float b,
                                float* x_next, cudaStream_t st) {
  const dit_config& c = H->cfg;
  const long long plane = static_cast<long long>(c.frames) * c.height * c.width;
  double c0 = 1.0, c1 = 0.0;
  if (kind == DIT_SAMPLER_DDIM) {
    const double da = a, db = b;
    c0 = std::sqrt(db / da);
    c1 = std::sqrt(1.0 - db) - std::sqrt(db) * std::sqrt(1.0 - da) / std::sqrt(da);
  } else {
    c1 = static_cast<double>(b) - static_cast<double>(a);
  }
  SamplerArgs sa;
  sa.x = x;
  sa.pred = pred;
  sa.x_next = x_next;
  sa.n_sample = plane * c.in_channels;
  sa.ld_pred = plane * H->g.Cout;
  sa.B = B;
  sa.c0 = static_cast<float>(c0);
  sa.c1 = static_cast<float>(c1);
  DIT_LAUNCH(H, DIT_KERNEL_SAMPLER, st, launch_sampler_step(sa, H->num_sms, st), "sampler step");
  return DIT_OK;
}

dit_status check_sampler(dit_handle* H, int kind, int B, const float* levels, int n_levels) {
  if (B < 1 || B > H->cfg.max_batch) return fail(H, DIT_ERR_INVALID_ARG, "batch outside [1, max_batch]");
  if (kind != DIT_SAMPLER_DDIM && kind != DIT_SAMPLER_EULER) return fail(H, DIT_ERR_INVALID_ARG, "unknown sampler kind");
  for (int i = 0; i < n_levels; ++i) {
    const float v = levels[i];
    if (!std::isfinite(v)) return fail(H, DIT_ERR_INVALID_ARG, "sampler level is not finite");
    if (kind == DIT_SAMPLER_DDIM && !(v > 0.f && v <= 1.f)) return fail(H, DIT_ERR_INVALID_ARG, "DDIM level outside (0, 1]");
  }
  return DIT_OK;
}

// steps x (forward into the handle's output buffer, then the update in place on x)
dit_status run_sample_loop(dit_handle* H, int kind, float* x, const void* y, const RunPlan& p, int steps,
                           const std::vector<float>& levels, cudaStream_t st) {
  for (int i = 0; i < steps; ++i) {
    dit_status s = run_forward(H, x, H->t_sched + static_cast<size_t>(i) * p.B, y, p, H->cfg.depth, H->out_stage, st);
    if (s != DIT_OK) return s;
    s = enqueue_sampler_step(H, kind, x, H->out_stage, p.B, levels[i], levels[i + 1], x, st);
    if (s != DIT_OK) return s;
  }
  return DIT_OK;
}

}  // namespace

extern "C" {

dit_status dit_set_option(dit_handle* H, int option, int value) {
  if (H == nullptr) return DIT_ERR_INVALID_ARG;
  if (option == DIT_OPT_FORCE_GUIDANCE) {
    H->force_guidance = value != 0;
    return DIT_OK;
  }
  if (option == DIT_OPT_USE_GRAPH) {
    H->use_graph = value != 0;
    return DIT_OK;
  }
  if (option == DIT_OPT_OVERLAP_LAUNCH) {
    dit::g_pdl = value != 0;
    return DIT_OK;
  }
  if (option == DIT_OPT_CFG_CHANNELS) {
    if (value < 0) return fail(H, DIT_ERR_INVALID_ARG, "guided channel count must be >= 0");
    H->cfg_channels = value;
    return DIT_OK;
  }
  if (option == DIT_OPT_SPLIT_K) {
    if (value < 1 || value > 8) return fail(H, DIT_ERR_INVALID_ARG, "split-K must be 1..8");
    H->ksplit_short = value;
    H->has_gseen = H->has_sseen = false;  // a new kernel configuration: recapture
    if (H->gexec != nullptr) cudaGraphExecDestroy(H->gexec);
    if (H->sexec != nullptr) cudaGraphExecDestroy(H->sexec);
    H->gexec = H->sexec = nullptr;
    return DIT_OK;
  }
  if (option == DIT_OPT_PAIR_GEMM) {
    H->pair_gemm = value != 0;
    H->has_gseen = H->has_sseen = false;  // a new kernel configuration: recapture
    if (H->gexec != nullptr) cudaGraphExecDestroy(H->gexec);
    if (H->sexec != nullptr) cudaGraphExecDestroy(H->sexec);
    H->gexec = H->sexec = nullptr;
    return DIT_OK;
  }
  if (option == DIT_OPT_REPEAT_KIND) {
    if (value < -1 || value >= DIT_KERNEL_COUNT) return fail(H, DIT_ERR_INVALID_ARG, "unknown kernel kind");
    H->repeat_kind = value;
    return DIT_OK;
  }

  return fail(H, DIT_ERR_INVALID_ARG, "unknown option");
}

dit_status dit_forward(dit_handle* H, const float* x, const float* t, const void* y, int B, float cfg_scale, float* out,
                       dit_stream_t stream) {
  RunPlan p;
  dit_status s = check_run(H, x, t, y, B, cfg_scale, p);
  if (s != DIT_OK) return s;
  if (out == nullptr) return fail(H, DIT_ERR_INVALID_ARG, "null output pointer");
  return run_forward_cached(H, x, t, y, p, out, reinterpret_cast<cudaStream_t>(stream));
}

dit_status dit_sampler_step(dit_handle* H, int kind, const float* x, const float* model_out, int B, float a, float b,
                            float* x_next, dit_stream_t stream) {
  if (H == nullptr) return DIT_ERR_INVALID_ARG;
  if (x == nullptr || model_out == nullptr || x_next == nullptr) return fail(H, DIT_ERR_INVALID_ARG, "null pointer");
  const float lv[2] = {a, b};
  dit_status s = check_sampler(H, kind, B, lv, 2);
  if (s != DIT_OK) return s;
  return enqueue_sampler_step(H, kind, x, model_out, B, a, b, x_next, reinterpret_cast<cudaStream_t>(stream));
}

dit_status dit_sample(dit_handle* H, int kind, float* x, const void* y, int B, float cfg_scale, int steps,
                      const float* model_t, const float* levels, dit_stream_t stream) {
  if (H == nullptr) return DIT_ERR_INVALID_ARG;
  if (steps < 1 || model_t == nullptr || levels == nullptr) return fail(H, DIT_ERR_INVALID_ARG, "bad step schedule");
  RunPlan p;
  dit_status s = check_run(H, x, model_t, y, B, cfg_scale, p);
  if (s != DIT_OK) return s;
  s = check_sampler(H, kind, B, levels, steps + 1);
  if (s != DIT_OK) return s;
  for (int i = 0; i < steps; ++i)
    if (!std::isfinite(model_t[i])) return fail(H, DIT_ERR_INVALID_ARG, "model timestep is not finite");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the per-step timestep of every sample, uploaded every call (outside any graph)
  const size_t need = static_cast<size_t>(steps) * B;
  if (need > H->t_sched_cap) {
    if (H->t_sched != nullptr) DIT_CK(H, cudaFree(H->t_sched), "timestep table");
    H->t_sched = nullptr;
    H->t_sched_cap = 0;
    DIT_CK(H, cudaMalloc(&H->t_sched, need * sizeof(float)), "timestep table");
    H->t_sched_cap = need;
  }
  H->t_host.assign(need, 0.f);
  for (int i = 0; i < steps; ++i)
    for (int b = 0; b < B; ++b) H->t_host[static_cast<size_t>(i) * B + b] = model_t[i];
  DIT_CK(H, cudaMemcpyAsync(H->t_sched, H->t_host.data(), need * sizeof(float), cudaMemcpyHostToDevice, st),
         "timestep upload");
  std::vector<float> lv(levels, levels + steps + 1);
  if (!H->use_graph || H->prof) return run_sample_loop(H, kind, x, y, p, steps, lv, st);
  dit_handle::SampleKey k;
  k.x = x;
  k.y = y;
  k.t_sched = H->t_sched;
  k.B = B;
  k.R = p.R;
  k.kind = kind;
  k.steps = steps;
  k.gch = H->cfg_channels;
  k.rep = H->repeat_kind;
  k.guided = p.guided;
  k.pdl = g_pdl;
  k.s = p.s;
  k.levels = lv;
  if (H->sexec != nullptr && k == H->skey) {
    DIT_CK(H, cudaGraphLaunch(H->sexec, st), "graph launch");
    return DIT_OK;
  }
  if (!(H->has_sseen && k == H->sseen)) {
    H->sseen = k;
    H->has_sseen = true;
    return run_sample_loop(H, kind, x, y, p, steps, lv, st);
  }
  if (H->cap_stream == nullptr) DIT_CK(H, cudaStreamCreateWithFlags(&H->cap_stream, cudaStreamNonBlocking), "capture stream");
  // the capture stream must see the timestep upload: it is ordered on `st`, so the graph
  // is launched on `st` after it; capturing itself records without executing.
  DIT_CK(H, cudaStreamBeginCapture(H->cap_stream, cudaStreamCaptureModeThreadLocal), "begin capture");
  const dit_status ls = run_sample_loop(H, kind, x, y, p, steps, lv, H->cap_stream);
  cudaGraph_t graph = nullptr;
  cudaError_t e = cudaStreamEndCapture(H->cap_stream, &graph);
  cudaGraphExec_t ex = nullptr;
  if (ls == DIT_OK && e == cudaSuccess) e = cudaGraphInstantiate(&ex, graph, 0);
  if (graph != nullptr) cudaGraphDestroy(graph);
  if (ls != DIT_OK || e != cudaSuccess || ex == nullptr) {
    cudaGetLastError();
    H->use_graph = 0;
    if (ls != DIT_OK) return ls;
    return run_sample_loop(H, kind, x, y, p, steps, lv, st);
  }
  if (H->sexec != nullptr) cudaGraphExecDestroy(H->sexec);
  H->sexec = ex;
  H->skey = k;
  DIT_CK(H, cudaGraphLaunch(H->sexec, st), "graph launch");
  return DIT_OK;
}

dit_status dit_forward_host(dit_handle* H, const float* x, const float* t, const void* y, int B, float cfg_scale,
                            float* out, dit_stream_t stream) {
  RunPlan p;
  dit_status s = check_run(H, x, t, y, B, cfg_scale, p);
  if (s != DIT_OK) return s;
  if (out == nullptr) return fail(H, DIT_ERR_INVALID_ARG, "null output pointer");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dit_config& c = H->cfg;
  const size_t xin = (size_t)B * c.in_channels * c.frames * c.height * c.width;
  const size_t xout = (size_t)B * H->g.Cout * c.frames * c.height * c.width;
  const size_t ybytes = (size_t)B * (c.cond_kind == DIT_COND_CLASS ? 4 : (size_t)c.hidden * 4);
  DIT_CK(H, cudaMemcpyAsync(H->x_stage, x, xin * 4, cudaMemcpyHostToDevice, st), "x upload");
  DIT_CK(H, cudaMemcpyAsync(H->t_stage, t, (size_t)B * 4, cudaMemcpyHostToDevice, st), "t upload");
  DIT_CK(H, cudaMemcpyAsync(H->y_stage, y, ybytes, cudaMemcpyHostToDevice, st), "y upload");
  s = run_forward_cached(H, H->x_stage, H->t_stage, H->y_stage, p, H->out_stage, st);
  if (s != DIT_OK) return s;
  DIT_CK(H, cudaMemcpyAsync(out, H->out_stage, xout * 4, cudaMemcpyDeviceToHost, st), "out download");
  DIT_CK(H, cudaStreamSynchronize(st), "stream sync");
  return DIT_OK;
}

dit_status dit_debug_residual(dit_handle* H, const float* x, const float* t, const void* y, int B, float cfg_scale,
                              int after_block, float* h_out, dit_stream_t stream) {
  RunPlan p;
  dit_status s = check_run(H, x, t, y, B, cfg_scale, p);
  if (s != DIT_OK) return s;
  if (h_out == nullptr || after_block < 0 || after_block > H->cfg.depth)
    return fail(H, DIT_ERR_INVALID_ARG, "bad residual request");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  s = run_forward(H, x, t, y, p, after_block, nullptr, st);
  if (s != DIT_OK) return s;
  DIT_CK(H, cudaMemcpyAsync(h_out, H->h, (size_t)p.M * H->cfg.hidden * 4, cudaMemcpyDeviceToDevice, st), "copy h");
  return DIT_OK;
}

dit_status dit_debug_condition(dit_handle* H, const float* t, const void* y, int B, float cfg_scale, float* c_out,
                               dit_stream_t stream) {
  RunPlan p;
  dit_status s = check_run(H, t, t, y, B, cfg_scale, p);
  if (s != DIT_OK) return s;
  if (c_out == nullptr) return fail(H, DIT_ERR_INVALID_ARG, "null output pointer");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  s = run_condition(H, t, y, p, st);
  if (s != DIT_OK) return s;
  DIT_CK(H, cudaMemcpyAsync(c_out, H->c, (size_t)p.R * H->cfg.hidden * 4, cudaMemcpyDeviceToDevice, st), "copy c");
  return DIT_OK;
}

dit_status dit_sync_status(dit_handle* H) {
  if (H == nullptr) return DIT_ERR_INVALID_ARG;
  DIT_CK(H, cudaDeviceSynchronize(), "sync");
  int v = 0;
  DIT_CK(H, cudaMemcpy(&v, H->status, 4, cudaMemcpyDeviceToHost), "status read");
  DIT_CK(H, cudaMemset(H->status, 0, 4), "status clear");
  return static_cast<dit_status>(v);
}

dit_status dit_debug_wait_probe(dit_handle* H, int timeout_us, dit_stream_t stream) {
  if (H == nullptr || timeout_us < 0) return DIT_ERR_INVALID_ARG;
  DIT_CK(H, launch_wait_probe(H->probe_flag, H->status, (long long)timeout_us * 1000LL,
                              reinterpret_cast<cudaStream_t>(stream)),
         "wait probe");
  return DIT_OK;
}

dit_status dit_profile_enable(dit_handle* H, int enable) {
  if (H == nullptr) return DIT_ERR_INVALID_ARG;
  if (enable < 0 || enable >= 2 + DIT_KERNEL_COUNT) return fail(H, DIT_ERR_INVALID_ARG, "bad profiling mode");
  H->prof = enable != 0;
  H->prof_kind = enable >= 2 ? enable - 2 : -1;
  return DIT_OK;
}

dit_status dit_profile_read(dit_handle* H, float* total_ms, int* launches) {
  if (H == nullptr || total_ms == nullptr || launches == nullptr) return DIT_ERR_INVALID_ARG;
  DIT_CK(H, cudaDeviceSynchronize(), "sync");
  for (int k = 0; k < DIT_KERNEL_COUNT; ++k) {
    total_ms[k] = 0.f;
    launches[k] = 0;
  }
  for (const auto& r : H->prof_recs) {
    float ms = 0.f;
    DIT_CK(H, cudaEventElapsedTime(&ms, H->ev_pool[r.second], H->ev_pool[r.second + 1]), "event time");
    if (r.first >= 0 && r.first < DIT_KERNEL_COUNT) {
      total_ms[r.first] += ms;
      launches[r.first] += 1;
    }
  }
  H->prof_recs.clear();
  return DIT_OK;
}

static dit_status op_linear(const uint16_t* x, const uint16_t* w, const float* b, float* y, int M, int N, int K,
                            int block_n, bool pair, cudaStream_t st) {
  if (x == nullptr || w == nullptr || y == nullptr || M < 0 || N <= 0 || K <= 0 || (K % 8) != 0)
    return DIT_ERR_INVALID_ARG;
  if (!(pair ? gemm_tc2_supported_bn(block_n) : gemm_tc_supported_bn(block_n))) return DIT_ERR_INVALID_ARG;
  if (M == 0) return DIT_OK;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DIT_ERR_NO_DEVICE;
  CUtensorMap ta, tb;
  if (!make_tmap_bf16_kmajor(&ta, x, M, K, 128) || !make_tmap_bf16_kmajor(&tb, w, N, K, pair ? block_n / 2 : block_n))
    return DIT_ERR_INVALID_ARG;
  EpiArgs ea = {};
  ea.M = M;
  ea.N = N;
  ea.bias = b;
  ea.out = y;
  ea.ldo = N;
  const cudaError_t e = pair ? launch_gemm_tc2(EPI_F32, block_n, &ta, &tb, K, ea, sms, st)
                             : launch_gemm_tc(EPI_F32, block_n, &ta, &tb, K, ea, sms, st);
  return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_op_linear_e4m3(const uint8_t* x, const uint8_t* w, const float* sx, const float* sw, const float* b,
                              float* y, int M, int N, int K, int block_n, dit_stream_t stream) {
  if (x == nullptr || w == nullptr || sx == nullptr || sw == nullptr || y == nullptr || M < 0 || N <= 0 || K <= 0 ||
      (K % 16) != 0)
    return DIT_ERR_INVALID_ARG;
  if (block_n != 64 && block_n != 128 && block_n != 256) return DIT_ERR_INVALID_ARG;
  if (M == 0) return DIT_OK;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DIT_ERR_NO_DEVICE;
  CUtensorMap ta, tb;
  if (!make_tmap_e4m3_kmajor(&ta, x, M, K, 128) || !make_tmap_e4m3_kmajor(&tb, w, N, K, block_n))
    return DIT_ERR_INVALID_ARG;
  EpiArgs ea = {};
  ea.M = M;
  ea.N = N;
  ea.bias = b;
  ea.out = y;
  ea.ldo = N;
  ea.sa = sx;
  ea.sb = sw;
  return launch_gemm_tc(EPI_F32_8, block_n, &ta, &tb, K, ea, sms, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DIT_OK
             : DIT_ERR_CUDA;
}

dit_status dit_op_attention_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* o, int R, int H,
                                 int T, int dh, int* counters, dit_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || R < 0 || H <= 0 || T <= 0)
    return DIT_ERR_INVALID_ARG;
  if (dh != 64 && dh != 72) return DIT_ERR_UNSUPPORTED;
  if (R == 0) return DIT_OK;
  const int DP = (dh + 15) / 16 * 16, Tpad = (T + 127) / 128 * 128, d = H * dh;
  AttnMaps maps;
  if (!make_attention_maps(&maps, q, k, v, o, R, H, T, Tpad, dh, DP, d)) return DIT_ERR_INVALID_ARG;
  AttnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.R = R;
  a.H = H;
  a.T = T;
  a.dh = dh;
  a.DP = DP;
  a.Tpad = Tpad;
  a.d = d;
  a.bf16 = 1;
  return launch_attention_tc(a, maps, counters, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? DIT_OK
                                                                                                         : DIT_ERR_CUDA;
}

dit_status dit_debug_attention_rescales(dit_handle* H, long long* count) {
  if (H == nullptr || count == nullptr) return DIT_ERR_INVALID_ARG;
  DIT_CK(H, cudaDeviceSynchronize(), "sync");
  int v = 0;
  DIT_CK(H, cudaMemcpy(&v, H->status + 1, 4, cudaMemcpyDeviceToHost), "counter read");
  DIT_CK(H, cudaMemset(H->status + 1, 0, 4), "counter clear");
  *count = v;
  return DIT_OK;
}

dit_status dit_op_linear_bf16_pair(const uint16_t* x, const uint16_t* w, const float* b, float* y, int M, int N, int K,
                                   int block_n, dit_stream_t stream) {
  return op_linear(x, w, b, y, M, N, K, block_n, true, reinterpret_cast<cudaStream_t>(stream));
}

dit_status dit_op_linear_bf16(const uint16_t* x, const uint16_t* w, const float* b, float* y, int M, int N, int K,
                              int block_n, dit_stream_t stream) {
  return op_linear(x, w, b, y, M, N, K, block_n, false, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
