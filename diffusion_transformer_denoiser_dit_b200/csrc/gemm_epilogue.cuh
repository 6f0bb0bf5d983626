// Fused epilogues of the tensor-core GEMMs.
//
// Eight epilogue warps per CTA: warp w reads TMEM lanes 32*(w%4)..+31 (one output
// row per thread) and one half of the tile's columns.  Columns are read from TMEM in
// chunks with tcgen05.ld; the load of chunk c+1 is in flight while chunk c is
// processed (tcgen05.wait::ld only after the processing), so TMEM latency overlaps
// the arithmetic and the global-memory traffic of the previous chunk.
// Epilogues: bias (+ tanh-GELU) to bf16, gated residual update of the float32
// stream, modulation-vector scatter, head-major Q / K / V^T scatter (swapped, or per
// whole head with QK-RMSNorm and 3D RoPE), plain float32 output.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace dit {

template <int W>
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, uint32_t* r) {
  if constexpr (W == 32) {
    tmem_ld32(taddr, r);
  } else if constexpr (W == 16) {
    tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
  } else {
    static_assert(W == 8, "chunk width");
    DIT_TMEM_LD_X8(taddr, r);
  }
}

// Columns [n, n + W) of output row m from the registers v (already accumulated).
template <int W, int EPI>
__device__ __forceinline__ void epilogue_chunk(const EpiArgs& ea, const uint32_t* r, int m, int n) {
  if (m >= ea.M || n >= ea.N) return;
  const bool full = n + W <= ea.N;
  if constexpr (EPI == EPI_ADALN) {
    // rows of this GEMM are modulation features j = m, columns are sample rows
    const float bj = __ldg(ea.bias + m);
    float* o = static_cast<float*>(ea.out) + m;
#pragma unroll
    for (int i = 0; i < W; ++i)
      if (n + i < ea.N) o[static_cast<size_t>(n + i) * ea.ldo] = __uint_as_float(r[i]) + bj;
  } else if constexpr (EPI == EPI_F32) {
    float* o = static_cast<float*>(ea.out) + static_cast<size_t>(m) * ea.ldo + n;
    if (full && (ea.ldo & 3) == 0) {
#pragma unroll
      for (int i = 0; i < W / 4; ++i) {
        const float4 b4 =
            ea.bias ? __ldg(reinterpret_cast<const float4*>(ea.bias + n) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(o)[i] =
            make_float4(__uint_as_float(r[4 * i]) + b4.x, __uint_as_float(r[4 * i + 1]) + b4.y,
                        __uint_as_float(r[4 * i + 2]) + b4.z, __uint_as_float(r[4 * i + 3]) + b4.w);
      }
    } else {
      for (int i = 0; i < W && n + i < ea.N; ++i) o[i] = __uint_as_float(r[i]) + (ea.bias ? __ldg(ea.bias + n + i) : 0.f);
    }
  } else if constexpr (EPI == EPI_F32_8) {
    const float sm = __ldg(ea.sa + m);
    float* o = static_cast<float*>(ea.out) + static_cast<size_t>(m) * ea.ldo + n;
    for (int i = 0; i < W && n + i < ea.N; ++i)
      o[i] = __uint_as_float(r[i]) * sm * __ldg(ea.sb + n + i) + (ea.bias ? __ldg(ea.bias + n + i) : 0.f);
  }
}

// One whole head (DH columns) of q, k or v for output row m: bias, optional
// QK-RMSNorm and 3D RoPE, head-major store.  FP8: E4M3 operands, the accumulator is first
// scaled by the token's scale sa[m] and each weight row's scale sb[n + j].
template <int DH, bool FP8 = false>
__device__ __forceinline__ void epilogue_head(const EpiArgs& ea, const uint32_t* r, int m, int n) {
  if (n >= ea.N) return;
  const int which = n / ea.d;
  const int head = (n - which * ea.d) / DH;
  const int row = m / ea.T, tok = m - row * ea.T;
  const float sm = FP8 && m < ea.M ? __ldg(ea.sa + m) : 1.f;
  float v[DH];
#pragma unroll
  for (int j = 0; j < DH; ++j) {
    const float acc = FP8 ? __uint_as_float(r[j]) * sm * __ldg(ea.sb + n + j) : __uint_as_float(r[j]);
    v[j] = acc + __ldg(ea.bias + n + j);
  }
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
    if (m < ea.M) {
      uint16_t* dst = static_cast<uint16_t*>(which == 0 ? ea.q : ea.k) +
                      (static_cast<size_t>(row * ea.H + head) * ea.Tpad + tok) * ea.DP;
#pragma unroll
      for (int c = 0; c < DH / 8; ++c)
        *reinterpret_cast<uint4*>(dst + c * 8) =
            make_uint4(pack_bf16x2(v[c * 8 + 0], v[c * 8 + 1]), pack_bf16x2(v[c * 8 + 2], v[c * 8 + 3]),
                       pack_bf16x2(v[c * 8 + 4], v[c * 8 + 5]), pack_bf16x2(v[c * 8 + 6], v[c * 8 + 7]));
    }
  } else if (m < ea.M) {
    uint16_t* dst = static_cast<uint16_t*>(ea.v) + static_cast<size_t>(row * ea.H + head) * ea.DP * ea.Tpad + tok;
#pragma unroll
    for (int j = 0; j < DH; ++j) dst[static_cast<size_t>(j) * ea.Tpad] = f32_to_bf16(v[j]);
  }
}

// Cross-attention of one token onto the two condition tokens of its row, for one head,
// fused into the query projection: q = acc + bias over the head's DH columns (n is the
// head's first column, a multiple of DH), scores s_k = q . key_k / sqrt(DH) for k = 0, 1,
// softmax, and o = p_0 value_0 + p_1 value_1 written as bf16 to xo[m, n .. n + DH).
template <int DH>
__device__ __forceinline__ void epilogue_xattn(const EpiArgs& ea, const uint32_t* r, int m, int n) {
  if (n >= ea.N || m >= ea.M) return;
  const int row = m / ea.T;
  const float4* k0 = reinterpret_cast<const float4*>(ea.xkv + static_cast<size_t>(2 * row) * ea.ld_xkv + n);
  const float4* k1 = reinterpret_cast<const float4*>(ea.xkv + static_cast<size_t>(2 * row + 1) * ea.ld_xkv + n);
  const float4* v0 = k0 + ea.d / 4;
  const float4* v1 = k1 + ea.d / 4;
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int j4 = 0; j4 < DH / 4; ++j4) {
    const float4 b4 = __ldg(reinterpret_cast<const float4*>(ea.bias + n) + j4);
    const float4 a = __ldg(k0 + j4), b = __ldg(k1 + j4);
    const float q0 = __uint_as_float(r[4 * j4 + 0]) + b4.x, q1 = __uint_as_float(r[4 * j4 + 1]) + b4.y;
    const float q2 = __uint_as_float(r[4 * j4 + 2]) + b4.z, q3 = __uint_as_float(r[4 * j4 + 3]) + b4.w;
    s0 = fmaf(q0, a.x, fmaf(q1, a.y, fmaf(q2, a.z, fmaf(q3, a.w, s0))));
    s1 = fmaf(q0, b.x, fmaf(q1, b.y, fmaf(q2, b.z, fmaf(q3, b.w, s1))));
  }
  const float sc = rsqrtf(static_cast<float>(DH));
  s0 *= sc;
  s1 *= sc;
  const float mx = fmaxf(s0, s1);
  const float e0 = expf(s0 - mx), e1 = expf(s1 - mx);
  const float inv = 1.0f / (e0 + e1);
  const float p0 = e0 * inv, p1 = e1 * inv;
  uint16_t* dst = static_cast<uint16_t*>(ea.xo) + static_cast<size_t>(m) * ea.d + n;
#pragma unroll
  for (int c = 0; c < DH / 8; ++c) {
    const float4 a0 = __ldg(v0 + 2 * c), a1 = __ldg(v0 + 2 * c + 1);
    const float4 b0 = __ldg(v1 + 2 * c), b1 = __ldg(v1 + 2 * c + 1);
    *reinterpret_cast<uint4*>(dst + c * 8) =
        make_uint4(pack_bf16x2(p0 * a0.x + p1 * b0.x, p0 * a0.y + p1 * b0.y),
                   pack_bf16x2(p0 * a0.z + p1 * b0.z, p0 * a0.w + p1 * b0.w),
                   pack_bf16x2(p0 * a1.x + p1 * b1.x, p0 * a1.y + p1 * b1.y),
                   pack_bf16x2(p0 * a1.z + p1 * b1.z, p0 * a1.w + p1 * b1.w));
  }
}

// The columns [n0 + c0, n0 + c0 + NC) of a tile for output row m; tacc addresses
// column 0 of the tile in this warp's TMEM lanes.
template <int NC, int EPI, bool HEADWISE>
__device__ __forceinline__ void epilogue_cols(const EpiArgs& ea, uint32_t tacc, int m, int n0, int c0) {
  if constexpr (HEADWISE) {
    // NC is exactly one head: load it whole (8-column loads), then process
    static_assert(NC % 8 == 0, "head width");
    uint32_t r[NC];
#pragma unroll
    for (int c = 0; c < NC / 8; ++c) DIT_TMEM_LD_X8(tacc + c0 + c * 8, (r + c * 8));
    tmem_ld_wait<NC>(r);
    if constexpr (EPI == EPI_XATTN)
      epilogue_xattn<NC>(ea, r, m, n0 + c0);
    else
      epilogue_head<NC, EPI == EPI_QKV_HEAD8>(ea, r, m, n0 + c0);
  } else {
    constexpr int W = NC % 32 == 0 ? 32 : (NC % 16 == 0 ? 16 : 8);
    constexpr int NCH = NC / W;
    uint32_t r[2][W];
    tmem_ld_chunk<W>(tacc + c0, r[0]);
    tmem_ld_wait<W>(r[0]);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      if (c + 1 < NCH) tmem_ld_chunk<W>(tacc + c0 + (c + 1) * W, r[(c + 1) & 1]);
      epilogue_chunk<W, EPI>(ea, r[c & 1], m, n0 + c0 + c * W);
      if (c + 1 < NCH) tmem_ld_wait<W>(r[(c + 1) & 1]);
    }
  }
}

// Epilogues that write through shared memory, each warp in its own 4 KB staging
// buffer: GELU and the swapped Q / K / V^T scatter stage 32 x 32 bf16 chunks and write
// them back out with plain coalesced 16-byte stores, whole 64-byte row segments instead
// of 32 scattered pieces per instruction; RESID_T stages [token][feature] boxes that one
// lane hands to the TMA unit as a float32 reduce-add into the residual stream, so the SM
// never reads the stream back (plain loads and stores of the stream, or red.global.add,
// slow the concurrent main loop more).
template <int EPI>
__host__ __device__ constexpr bool epi_staged() {
  return EPI == EPI_GELU || EPI == EPI_RESID_T || EPI == EPI_RESID_T8 || EPI == EPI_QKV_T || EPI == EPI_QKV_T8;
}
constexpr int kStageBytesPerWarp = 4096;
constexpr int kEpilogueWarps = 8;

// GELU epilogue through shared memory: two 32-column chunks (64 columns, 128 bytes of
// bf16 per row) are written to the warp's 4 KB staging buffer as 32 rows of 128 bytes, the
// 16-byte group g of row r stored at g ^ (r & 7) so that the lanes' row writes and the
// read-back both spread over all banks, then read back so that 8 consecutive lanes cover
// one whole 128-byte output line: each store instruction writes 4 full lines.  Whole
// lines keep the store requests the epilogue sends to L2 few, which matters because they
// share the SM's path to L2 with the main loop's TMA loads of the next tile.
template <int NC, int EPI>
__device__ __forceinline__ void epilogue_cols_staged(const EpiArgs& ea, uint32_t tacc, int m_base, int lane, int n0,
                                                     int c0, uint8_t* stg) {
  static_assert(EPI == EPI_GELU, "staged row-major epilogue is the GELU output");
  static_assert(NC % 64 == 0, "staged epilogues work on 64-column pieces");
  constexpr int NCH = NC / 32;
  uint32_t r[2][32];
  tmem_ld_chunk<32>(tacc + c0, r[0]);
  tmem_ld_wait<32>(r[0]);
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    if (c + 1 < NCH) tmem_ld_chunk<32>(tacc + c0 + (c + 1) * 32, r[(c + 1) & 1]);
    const int n = n0 + c0 + c * 32;
    const int h = c & 1;  // which half of the 64-column piece
    const uint32_t* v = r[c & 1];
    if (h == 0) __syncwarp();  // every lane is done reading the previous piece
    if (n < ea.N) {
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        const float4 b0 = __ldg(reinterpret_cast<const float4*>(ea.bias + n) + 2 * c16);
        const float4 b1 = __ldg(reinterpret_cast<const float4*>(ea.bias + n) + 2 * c16 + 1);
        const uint32_t* w = v + 8 * c16;
        uint4 pk;  // bias and GELU on column pairs (paired float32 instructions)
        pk.x = pack_bf16x2_f2(gelu_tanh_fast_f2(
            f2_add(f2_pack(__uint_as_float(w[0]), __uint_as_float(w[1])), f2_pack(b0.x, b0.y))));
        pk.y = pack_bf16x2_f2(gelu_tanh_fast_f2(
            f2_add(f2_pack(__uint_as_float(w[2]), __uint_as_float(w[3])), f2_pack(b0.z, b0.w))));
        pk.z = pack_bf16x2_f2(gelu_tanh_fast_f2(
            f2_add(f2_pack(__uint_as_float(w[4]), __uint_as_float(w[5])), f2_pack(b1.x, b1.y))));
        pk.w = pack_bf16x2_f2(gelu_tanh_fast_f2(
            f2_add(f2_pack(__uint_as_float(w[6]), __uint_as_float(w[7])), f2_pack(b1.z, b1.w))));
        *reinterpret_cast<uint4*>(stg + lane * 128 + (((h * 4 + c16) ^ (lane & 7)) << 4)) = pk;
      }
    }
    if (h == 1) {
      __syncwarp();
      const int np = n - 32;  // first column of the piece
#pragma unroll
      for (int it = 0; it < 8; ++it) {  // 4 rows x 128 bytes per instruction
        const int rr = it * 4 + (lane >> 3), g = lane & 7;
        const uint4 val = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((g ^ (rr & 7)) << 4));
        const int m = m_base + rr, col = np + g * 8;
        if (m < ea.M && col < ea.N)
          *reinterpret_cast<uint4*>(static_cast<uint16_t*>(ea.out) + static_cast<size_t>(m) * ea.ldo + col) = val;
      }
    }
    if (c + 1 < NCH) tmem_ld_wait<32>(r[(c + 1) & 1]);
  }
}

// Swapped-operand residual update: lane = output feature f (TMEM lane), columns =
// tokens.  16-token x 32-feature boxes are staged as [token][feature] float32 rows
// (128B swizzle: 16-byte group g of row t at g ^ (t & 7)) in two alternating 2 KB
// buffers, written one token row per instruction by the 32 lanes, and added into the
// residual stream by the TMA unit (cp.reduce.async.bulk .add), so the SM never reads
// the stream back.
// FP8 = true: E4M3 operands, the accumulator is first scaled by the weight row's scale sa[f]
// and each token's scale sb[tok].
// with_bias = false: a split-K slice other than the first adds its partial product only.
template <int NC, bool FP8 = false>
__device__ __forceinline__ void epilogue_resid_t(const EpiArgs& ea, const CUtensorMap* tmC, uint32_t tacc, int f_base,
                                                 int lane, int n0, int c0, uint8_t* stg, bool with_bias = true) {
  static_assert(NC % 32 == 0, "32-token chunks");
  constexpr int NCH = NC / 32;
  const int f = f_base + lane;
  const bool fok = f < ea.M;
  const float bf = (fok && with_bias) ? __ldg(ea.bias + f) : 0.f;
  const float sf = (FP8 && fok) ? __ldg(ea.sa + f) : 1.f;
  uint32_t r[2][32];
  tmem_ld_chunk<32>(tacc + c0, r[0]);
  tmem_ld_wait<32>(r[0]);
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    if (c + 1 < NCH) tmem_ld_chunk<32>(tacc + c0 + (c + 1) * 32, r[(c + 1) & 1]);
    const int tok0 = n0 + c0 + c * 32;
    const uint32_t* v = r[c & 1];
    if (tok0 < ea.N) {
      const int last = min(tok0 + 31, ea.N - 1);
      const int r0 = tok0 / ea.T, r1 = last / ea.T;
      const float g0 = fok ? __ldg(ea.gate + static_cast<size_t>(r0) * ea.ld_gate + f) : 0.f;
      // FP8: lane l holds token tok0 + l's scale, handed to every lane below
      const float st_l = FP8 ? (tok0 + lane < ea.N ? __ldg(ea.sb + tok0 + lane) : 0.f) : 1.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // 16 tokens per box, alternating 2 KB buffers
        uint8_t* buf = stg + half * 2048;
        if (lane == 0) bulk_wait_read_but1();
        __syncwarp();
#pragma unroll
        for (int tt = 0; tt < 16; tt += 2) {  // token pairs: paired float32 arithmetic
          const int t = half * 16 + tt;
          float ga = g0, gb = g0;
          if (r1 != r0) {
            const int ra = min(tok0 + t, ea.N - 1) / ea.T, rb = min(tok0 + t + 1, ea.N - 1) / ea.T;
            ga = fok ? __ldg(ea.gate + static_cast<size_t>(ra) * ea.ld_gate + f) : 0.f;
            gb = fok ? __ldg(ea.gate + static_cast<size_t>(rb) * ea.ld_gate + f) : 0.f;
          }
          uint64_t acc = f2_pack(__uint_as_float(v[t]), __uint_as_float(v[t + 1]));
          if constexpr (FP8)
            acc = f2_mul(acc, f2_pack(sf * __shfl_sync(0xffffffffu, st_l, t), sf * __shfl_sync(0xffffffffu, st_l, t + 1)));
          float ya, yb;
          f2_unpack(f2_mul(f2_add(acc, f2_pack(bf, bf)), f2_pack(ga, gb)), ya, yb);
          // [token][feature] float32 rows of 128 bytes, 128B swizzle
          *reinterpret_cast<float*>(buf + tt * 128 + ((((lane >> 2) ^ (tt & 7)) << 4) | ((lane & 3) << 2))) = ya;
          *reinterpret_cast<float*>(buf + (tt + 1) * 128 + ((((lane >> 2) ^ ((tt + 1) & 7)) << 4) | ((lane & 3) << 2))) =
              yb;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && f_base < ea.M && tok0 + half * 16 < ea.N) {
          tma_reduce_add_2d(tmC, smem_u32(buf), f_base, tok0 + half * 16);
          bulk_commit_group();
        }
      }
    }
    if (c + 1 < NCH) tmem_ld_wait<32>(r[(c + 1) & 1]);
  }
}

// FP8 feed-forward hidden layer: for output row m and columns [n0 + c0, n0 + c0 + NC),
// z = sa[m] sb[n] acc + bias[n], g = gelu_tanh(z), stored as E4M3 g / sg[m] (one byte per
// column; 32 columns leave as two 16-byte stores per thread).
template <int NC>
__device__ __forceinline__ void epilogue_gelu8(const EpiArgs& ea, uint32_t tacc, int m, int n0, int c0) {
  static_assert(NC % 32 == 0, "32-column chunks");
  constexpr int NCH = NC / 32;
  const bool mok = m < ea.M;
  const float sm = mok ? __ldg(ea.sa + m) : 0.f;
  const float inv = mok ? 1.0f / __ldg(ea.sg + m) : 0.f;
  uint32_t r[2][32];
  tmem_ld_chunk<32>(tacc + c0, r[0]);
  tmem_ld_wait<32>(r[0]);
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    if (c + 1 < NCH) tmem_ld_chunk<32>(tacc + c0 + (c + 1) * 32, r[(c + 1) & 1]);
    const int n = n0 + c0 + c * 32;
    const uint32_t* v = r[c & 1];
    if (mok && n < ea.N) {
      uint32_t pk[8];
#pragma unroll
      for (int i4 = 0; i4 < 8; ++i4) {
        const float4 s4 = __ldg(reinterpret_cast<const float4*>(ea.sb + n) + i4);
        const float4 b4 = __ldg(reinterpret_cast<const float4*>(ea.bias + n) + i4);
        // z = sm s acc + bias and GELU on column pairs (paired float32 instructions)
        const uint64_t sm2 = f2_pack(sm, sm), inv2 = f2_pack(inv, inv);
        const uint64_t za = f2_fma(f2_mul(f2_pack(__uint_as_float(v[4 * i4 + 0]), __uint_as_float(v[4 * i4 + 1])), sm2),
                                   f2_pack(s4.x, s4.y), f2_pack(b4.x, b4.y));
        const uint64_t zb = f2_fma(f2_mul(f2_pack(__uint_as_float(v[4 * i4 + 2]), __uint_as_float(v[4 * i4 + 3])), sm2),
                                   f2_pack(s4.z, s4.w), f2_pack(b4.z, b4.w));
        float g0, g1, g2, g3;
        f2_unpack(f2_mul(gelu_tanh_fast_f2(za), inv2), g0, g1);
        f2_unpack(f2_mul(gelu_tanh_fast_f2(zb), inv2), g2, g3);
        pk[i4] = pack_e4m3x4(g0, g1, g2, g3);
      }
      uint4* o = reinterpret_cast<uint4*>(static_cast<uint8_t*>(ea.out) + static_cast<size_t>(m) * ea.ldo + n);
      o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    if (c + 1 < NCH) tmem_ld_wait<32>(r[(c + 1) & 1]);
  }
}

// 32 consecutive tokens of one V^T row from registers, starting at a destination whose
// offset from a 16-byte boundary is (8 - A) % 8 tokens: A scalar stores reach the boundary,
// then 16-byte groups of 8 tokens, then the scalar tail.  A is a template argument so that the
// register array is indexed with constants.
template <int A>
__device__ __forceinline__ void store_vt_row32(uint16_t* dst, const uint32_t* v, float bf) {
#pragma unroll
  for (int t = 0; t < A; ++t) dst[t] = f32_to_bf16(__uint_as_float(v[t]) + bf);
#pragma unroll
  for (int g = 0; A + 8 * g + 8 <= 32; ++g) {
    const int t = A + 8 * g;
    *reinterpret_cast<uint4*>(dst + t) =
        make_uint4(pack_bf16x2(__uint_as_float(v[t + 0]) + bf, __uint_as_float(v[t + 1]) + bf),
                   pack_bf16x2(__uint_as_float(v[t + 2]) + bf, __uint_as_float(v[t + 3]) + bf),
                   pack_bf16x2(__uint_as_float(v[t + 4]) + bf, __uint_as_float(v[t + 5]) + bf),
                   pack_bf16x2(__uint_as_float(v[t + 6]) + bf, __uint_as_float(v[t + 7]) + bf));
  }
  constexpr int tail = A + (32 - A) / 8 * 8;
#pragma unroll
  for (int t = tail; t < 32; ++t) dst[t] = f32_to_bf16(__uint_as_float(v[t]) + bf);
}

// Swapped-operand Q / K / V^T scatter: lane = output feature f of [q | k | v],
// columns = tokens.  A chunk of 32 features x 32 tokens normally goes through the warp's
// staging buffer so that each global store instruction writes eight whole 64-byte
// segments: q and k are staged [token][feature] (one token's 32 features, contiguous in
// the head-major layout except at a head boundary, which falls between 16-byte groups
// because the head dim is a multiple of 8), V^T is staged [feature][token] (32
// consecutive tokens of one V^T row, 16-byte groups of row r rotated by (r >> 1) & 3).
// Chunks that straddle two sample rows, V^T chunks that start off a 16-byte boundary and
// widths d that are not a multiple of 32 are written lane by lane instead: V^T as 16-byte
// groups of 8 tokens, q and k one token per instruction.
// FP8 = true: E4M3 operands, the accumulator is first scaled by the weight row's scale sa[f]
// and each token's scale sb[tok].
template <int NC, bool FP8 = false>
__device__ __forceinline__ void epilogue_qkv_t(const EpiArgs& ea, uint32_t tacc, int f_base, int lane, int n0, int c0,
                                               uint8_t* stg) {
  static_assert(NC % 32 == 0, "32-token chunks");
  constexpr int NCH = NC / 32;
  const int f = f_base + lane;
  const bool fok = f < ea.M;
  const int which = fok ? f / ea.d : 0;
  const int within = f - which * ea.d;
  const int head = within / ea.dh, j = within - head * ea.dh;
  const float bf = fok ? __ldg(ea.bias + f) : 0.f;
  const float sf = (FP8 && fok) ? __ldg(ea.sa + f) : 1.f;
  uint16_t* qk = static_cast<uint16_t*>(which == 0 ? ea.q : ea.k);
  // staging: all 32 features of the warp are q, all k or all v
  const bool warp_one_kind = (ea.d & 31) == 0 && f_base + 31 < ea.M;
  int gh = 0, gj = 0;  // q / k read-back: head and offset of this lane's 8-feature group (lane & 3)
  int vh[4] = {0, 0, 0, 0}, vj[4] = {0, 0, 0, 0};  // V^T read-back: feature row it * 8 + (lane >> 2)
  if (warp_one_kind) {
    const int wbase = f_base - (f_base / ea.d) * ea.d;
    const int wg = wbase + 8 * (lane & 3);
    gh = wg / ea.dh;
    gj = wg - gh * ea.dh;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int wf = wbase + it * 8 + (lane >> 2);
      vh[it] = wf / ea.dh;
      vj[it] = wf - vh[it] * ea.dh;
    }
  }
  uint32_t r[2][32];
  tmem_ld_chunk<32>(tacc + c0, r[0]);
  tmem_ld_wait<32>(r[0]);
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    if (c + 1 < NCH) tmem_ld_chunk<32>(tacc + c0 + (c + 1) * 32, r[(c + 1) & 1]);
    const int tok0 = n0 + c0 + c * 32;
    uint32_t* v = r[c & 1];
    if constexpr (FP8) {
      if (tok0 < ea.N) {  // lane l holds token tok0 + l's scale, handed to every lane
        const float st_l = tok0 + lane < ea.N ? __ldg(ea.sb + tok0 + lane) : 0.f;
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = __float_as_uint(__uint_as_float(v[t]) * sf * __shfl_sync(0xffffffffu, st_l, t));
      }
    }
    if (fok && tok0 < ea.N) {
      const int last = min(tok0 + 31, ea.N - 1);
      const int r0 = tok0 / ea.T, t0 = tok0 - r0 * ea.T;
      const bool one_row = (last / ea.T) == r0 && last - tok0 == 31;
      if (warp_one_kind && one_row && (which < 2 || (t0 & 7) == 0)) {
        uint8_t* buf = stg + (c & 1) * 2048;
        const uint64_t bf2 = f2_pack(bf, bf);
        __syncwarp();  // every lane is done reading this buffer's previous chunk
        if (which == 2) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint32_t* w = v + 8 * g;
            *reinterpret_cast<uint4*>(buf + lane * 64 + ((g ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(pack_bf16x2_f2(f2_add(f2_pack(__uint_as_float(w[0]), __uint_as_float(w[1])), bf2)),
                           pack_bf16x2_f2(f2_add(f2_pack(__uint_as_float(w[2]), __uint_as_float(w[3])), bf2)),
                           pack_bf16x2_f2(f2_add(f2_pack(__uint_as_float(w[4]), __uint_as_float(w[5])), bf2)),
                           pack_bf16x2_f2(f2_add(f2_pack(__uint_as_float(w[6]), __uint_as_float(w[7])), bf2)));
          }
          __syncwarp();
          uint16_t* vb = static_cast<uint16_t*>(ea.v) + static_cast<size_t>(r0 * ea.H) * ea.DP * ea.Tpad + t0 +
                         8 * (lane & 3);
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int rr = it * 8 + (lane >> 2), g = lane & 3;
            const uint4 val = *reinterpret_cast<const uint4*>(buf + rr * 64 + ((g ^ ((rr >> 1) & 3)) << 4));
            *reinterpret_cast<uint4*>(vb + (static_cast<size_t>(vh[it]) * ea.DP + vj[it]) * ea.Tpad) = val;
          }
        } else {
#pragma unroll
          for (int t = 0; t < 32; t += 2) {  // bias and conversion on token pairs, one row each
            const uint32_t p = pack_bf16x2_f2(f2_add(f2_pack(__uint_as_float(v[t]), __uint_as_float(v[t + 1])), bf2));
            *reinterpret_cast<uint16_t*>(buf + t * 64 + lane * 2) = static_cast<uint16_t>(p & 0xffffu);
            *reinterpret_cast<uint16_t*>(buf + (t + 1) * 64 + lane * 2) = static_cast<uint16_t>(p >> 16);
          }
          __syncwarp();
          uint16_t* qb = qk + (static_cast<size_t>(r0 * ea.H + gh) * ea.Tpad + t0) * ea.DP + gj;
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int tt = it * 8 + (lane >> 2);
            *reinterpret_cast<uint4*>(qb + static_cast<size_t>(tt) * ea.DP) =
                *reinterpret_cast<const uint4*>(buf + tt * 64 + (lane & 3) * 16);
          }
        }
      } else if (which == 2) {
        if (one_row) {  // V^T row segment of 32 tokens: 16-byte groups from the first aligned token on
          uint16_t* dst = static_cast<uint16_t*>(ea.v) + (static_cast<size_t>(r0 * ea.H + head) * ea.DP + j) * ea.Tpad + t0;
          switch ((8 - (t0 & 7)) & 7) {
            case 0: store_vt_row32<0>(dst, v, bf); break;
            case 1: store_vt_row32<1>(dst, v, bf); break;
            case 2: store_vt_row32<2>(dst, v, bf); break;
            case 3: store_vt_row32<3>(dst, v, bf); break;
            case 4: store_vt_row32<4>(dst, v, bf); break;
            case 5: store_vt_row32<5>(dst, v, bf); break;
            case 6: store_vt_row32<6>(dst, v, bf); break;
            default: store_vt_row32<7>(dst, v, bf); break;
          }
        } else if (ea.T < 32) {  // short rows: a chunk spans several sample rows
          for (int t = 0; t < 32 && tok0 + t < ea.N; ++t) {
            const int rt = (tok0 + t) / ea.T, tt = tok0 + t - rt * ea.T;
            static_cast<uint16_t*>(ea.v)[(static_cast<size_t>(rt * ea.H + head) * ea.DP + j) * ea.Tpad + tt] =
                f32_to_bf16(__uint_as_float(v[t]) + bf);
          }
        } else {  // the chunk crosses into the next sample row (or the end): split once, no divides
          const int b = ea.T - t0;  // tokens of row r0 in the chunk
          uint16_t* d0 = static_cast<uint16_t*>(ea.v) + (static_cast<size_t>(r0 * ea.H + head) * ea.DP + j) * ea.Tpad + t0;
          uint16_t* d1 = static_cast<uint16_t*>(ea.v) + (static_cast<size_t>((r0 + 1) * ea.H + head) * ea.DP + j) * ea.Tpad;
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            if (tok0 + t >= ea.N) break;
            const uint16_t val = f32_to_bf16(__uint_as_float(v[t]) + bf);
            if (t < b)
              d0[t] = val;
            else
              d1[t - b] = val;
          }
        }
      } else {
        if (one_row) {
          uint16_t* dst = qk + (static_cast<size_t>(r0 * ea.H + head) * ea.Tpad + t0) * ea.DP + j;
#pragma unroll
          for (int t = 0; t < 32; ++t) dst[static_cast<size_t>(t) * ea.DP] = f32_to_bf16(__uint_as_float(v[t]) + bf);
        } else if (ea.T < 32) {  // short rows: a chunk spans several sample rows
          for (int t = 0; t < 32 && tok0 + t < ea.N; ++t) {
            const int rt = (tok0 + t) / ea.T, tt = tok0 + t - rt * ea.T;
            qk[(static_cast<size_t>(rt * ea.H + head) * ea.Tpad + tt) * ea.DP + j] = f32_to_bf16(__uint_as_float(v[t]) + bf);
          }
        } else {  // the chunk crosses into the next sample row (or the end): split once, no divides
          const int b = ea.T - t0;
          uint16_t* d0 = qk + (static_cast<size_t>(r0 * ea.H + head) * ea.Tpad + t0) * ea.DP + j;
          uint16_t* d1 = qk + static_cast<size_t>((r0 + 1) * ea.H + head) * ea.Tpad * ea.DP + j;
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            if (tok0 + t >= ea.N) break;
            const uint16_t val = f32_to_bf16(__uint_as_float(v[t]) + bf);
            if (t < b)
              d0[static_cast<size_t>(t) * ea.DP] = val;
            else
              d1[static_cast<size_t>(t - b) * ea.DP] = val;
          }
        }
      }
    }
    if (c + 1 < NCH) tmem_ld_wait<32>(r[(c + 1) & 1]);
  }
}

}  // namespace dit
