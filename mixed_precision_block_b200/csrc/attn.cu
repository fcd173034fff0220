// Stage 3: mixed-precision block-sparse attention with the output restored to
// token order, and the own dense bf16 attention used as the comparison point.
//
// DraftAttention2 abstract and reading note (Method overview bullet 4): one
// kernel runs a phase per precision for each query block; the phases share
// data movement, the softmax statistics and one output accumulator, and the
// quantisation scales are applied when a block is merged, so partial outputs
// are never written back and merged.  DraftAttention (v1) abstract: tokens are
// restored to their original order after attention — done here in the
// epilogue, which writes each block row straight to its token.
//
// attn_mp: one CTA (4 warps, 16 query rows each) per (query block, head).
//   phase 16  bf16 Q/K/V tiles gathered from the [B,H,N,d] inputs (8 rows of 8
//             contiguous tokens per region), cp.async double-buffered,
//             m16n8k16 bf16 MMAs, online softmax, P in bf16.
//   The low-bit phases walk the key blocks in units of two, as the
//   tensor-core kernel does for the query-block pair (2p, 2p+1): per unit the
//   row maximum over the member blocks comes first (scores only), raising the
//   phase's power-of-two P reference 2^r to ceil(max) where the max exceeds
//   it; then each member block is scored again and its P quantised against 2^r.
//   phase 8   INT8 Q/K codes with block scales (m16n8k32 s8·s8 → s32);
//             P = round(255·2^(x − r)) as u8 through shared memory;
//             P·V on u8·s8 codes; int32 block result scaled by
//             2^(r − m)/255 and the per-channel V scale when merged.
//   phase 4   NVFP4 codes dequantised exactly to f16 in shared memory
//             (e2m1 × e4m3 fits f16), m16n8k16 f16 MMAs, 2688·P
//             re-quantised to NVFP4 per 16 keys in registers, block result
//             scaled by 2^(r − m)/2688 and the per-channel V scale g when merged.
// attn_dense: the phase-16 path over all tokens in natural order.
#include "da2_internal.cuh"
#include "mma_sm80.cuh"

namespace da2 {
namespace {

constexpr int kWarps = 4;
constexpr int kAttnThreads = kWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct SmemLayout {
  static constexpr int TILE16 = 64 * D * 2;  // one bf16/f16 [64][D] tile
  static constexpr int Q = 0;
  static constexpr int K = Q + TILE16;       // 2 stages
  static constexpr int V = K + 2 * TILE16;   // 2 stages
  static constexpr int RAW = V + 2 * TILE16; // 2 stages of NVFP4 codes + scales
  static constexpr int KSF = (D / 64) * kSfAtomBytes;  // K scales of one block
  static constexpr int RAW_KC = 0, RAW_KS = 64 * D / 2, RAW_VC = RAW_KS + KSF,
                       RAW_VS = RAW_VC + D * 32, RAW_STAGE = RAW_VS + kSfAtomBytes;
  static constexpr int P = RAW + 2 * RAW_STAGE;  // per warp [16][64] u8
  static constexpr int VS = P + kWarps * 1024;   // per-channel V scale (fp32)
  static constexpr int TOTAL = VS + D * 4;
};

struct AttnArgs {
  const __nv_bfloat16 *q, *k, *v;
  __nv_bfloat16* out;
  const int8_t *q_i8, *k_i8, *v_i8;
  const float *q_s8, *k_s8, *v_s8;
  const uint8_t *q_f4, *k_f4, *q_sf4, *k_sf4, *v_f4, *v_sf4;
  const float* v_g4;
  const uint16_t* lists;
  const int* counts;
  const uint32_t* plist;  // merged key lists of the query-block pairs
  const int* pcnt;
};

// Real-token mask of a region block's 64 slots.
__device__ __forceinline__ unsigned long long region_mask(const Geom& g, int blk) {
  const int rx = blk % g.nrx;
  const int ry = (blk / g.nrx) % g.nry;
  const int vy = min(g.rh, g.Hh - ry * g.rh), vx = min(g.rw, g.Ww - rx * g.rw);
  const unsigned long long rowbits = (vx >= 64) ? ~0ull : ((1ull << vx) - 1ull);
  unsigned long long m = 0;
  for (int i = 0; i < vy; ++i) m |= rowbits << (g.rw * i);
  return m;
}

// cp.async of a bf16 [64][D] tile whose row r lives at src + tok(r)*D
// (tok < 0: zero row) into a swizzled shared tile.
template <int D, typename TokFn>
__device__ __forceinline__ void load_rows_bf16(uint32_t dst, const __nv_bfloat16* src, TokFn tok) {
  constexpr int CPR = D / 8;
  for (int e = threadIdx.x; e < 64 * CPR; e += kAttnThreads) {
    const int r = e / CPR, c = e % CPR;
    const int t = tok(r);
    const __nv_bfloat16* p = t >= 0 ? src + (size_t)t * D + c * 8 : src;
    cp_async16(dst + swz<CPR>(r, c), p, t >= 0 ? 16 : 0);
  }
}

// cp.async of a contiguous byte tile [rows][RB] into a swizzled shared tile.
template <int RB>
__device__ __forceinline__ void load_bytes_swz(uint32_t dst, const uint8_t* src, int rows) {
  constexpr int CPR = RB / 16;
  for (int e = threadIdx.x; e < rows * CPR; e += kAttnThreads) {
    const int r = e / CPR, c = e % CPR;
    cp_async16(dst + swz<CPR>(r, c), src + (size_t)r * RB + c * 16, 16);
  }
}

// cp.async of a contiguous run of bytes (multiple of 16) without swizzle.
__device__ __forceinline__ void load_bytes(uint32_t dst, const uint8_t* src, int bytes) {
  for (int e = threadIdx.x; e < bytes / 16; e += kAttnThreads)
    cp_async16(dst + e * 16, src + e * 16, 16);
}

// Dequantise an NVFP4 tile (codes [rows][cols/2], e4m3 scales in the atom layout)
// to f16 [rows][cols] in a swizzled shared tile.  Every value e2m1 × e4m3 is
// exact in f16.  `codes`/`scales` may be global or shared (generic pointers).
template <int COLS>
__device__ __forceinline__ void dequant_f4_tile(uint8_t* dst, const uint8_t* codes,
                                                const uint8_t* scales, int rows) {
  constexpr int CPR = COLS / 8;  // 16-byte f16 chunks per row = 8 values
  for (int e = threadIdx.x; e < rows * CPR; e += kAttnThreads) {
    const int r = e / CPR, c = e % CPR;
    const uint32_t w = *reinterpret_cast<const uint32_t*>(codes + (size_t)r * (COLS / 2) + c * 4);
    const uint32_t sb = scales[sf_atom_offset(r, c / 2)];
    uint32_t h2;
    {
      const uint16_t b = (uint16_t)(sb | (sb << 8));
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(b));
    }
    const __half2 s2 = *reinterpret_cast<const __half2*>(&h2);
    uint4 out;
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t v = e2m1x2_to_f16x2((w >> (8 * i)) & 0xffu);
      __half2 hv = __hmul2(*reinterpret_cast<__half2*>(&v), s2);
      o[i] = *reinterpret_cast<uint32_t*>(&hv);
    }
    *reinterpret_cast<uint4*>(dst + swz<CPR>(r, c)) = out;
  }
}

// S = Q K^T for this warp's 16 rows × 64 keys, 16-bit operands.
template <int D, bool F16>
__device__ __forceinline__ void qk_16bit(uint32_t sQ, uint32_t sK, int warp, int lane, float (*S)[4]) {
  constexpr int CPR = D / 8;
#pragma unroll
  for (int j = 0; j < 8; ++j) S[j][0] = S[j][1] = S[j][2] = S[j][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(sQ + swz<CPR>(warp * 16 + (lane & 15), 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sK + swz<CPR>(16 * np + (lane & 7) + ((lane >> 4) << 3), 2 * kk + ((lane >> 3) & 1)),
              b0, b1, b2, b3);
      if (F16) { mma_f16(S[2 * np], a, b0, b1); mma_f16(S[2 * np + 1], a, b2, b3); }
      else { mma_bf16(S[2 * np], a, b0, b1); mma_bf16(S[2 * np + 1], a, b2, b3); }
    }
  }
}

// Scale to log2 units and mask padding keys; returns the two row maxima.
__device__ __forceinline__ void scale_mask(float (*S)[4], float sc, unsigned long long vmask, int tq,
                                          float& mx0, float& mx1) {
  mx0 = mx1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int key = 8 * j + 2 * tq + e;
      const bool ok = (vmask >> key) & 1ull;
      S[j][e] = ok ? S[j][e] * sc : -INFINITY;
      S[j][2 + e] = ok ? S[j][2 + e] * sc : -INFINITY;
      mx0 = fmaxf(mx0, S[j][e]);
      mx1 = fmaxf(mx1, S[j][2 + e]);
    }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
}

__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

// One bf16 key block: online softmax update and O += P V (V row-major tile).
template <int D>
__device__ __forceinline__ void block16(uint32_t sQ, uint32_t sK, uint32_t sV, unsigned long long vmask,
                                        float sl2, int warp, int lane, float (*O)[4], float* m,
                                        float* l) {
  constexpr int CPR = D / 8;
  const int tq = lane & 3;
  float S[8][4];
  qk_16bit<D, false>(sQ, sK, warp, lane, S);
  float mx0, mx1;
  scale_mask(S, sl2, vmask, tq, mx0, mx1);
  // the reference is the running max rounded up to an integer exponent, so
  // P's bf16 rounding is relative to a power of two and rescales are exact
  const float mn0 = fmaxf(m[0], ceilf(mx0)), mn1 = fmaxf(m[1], ceilf(mx1));
  const float al0 = m[0] == -INFINITY ? 0.f : ldexpf(1.0f, (int)(m[0] - mn0));
  const float al1 = m[1] == -INFINITY ? 0.f : ldexpf(1.0f, (int)(m[1] - mn1));
  m[0] = mn0; m[1] = mn1;
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    S[j][0] = fast_exp2(S[j][0] - mn0); S[j][1] = fast_exp2(S[j][1] - mn0);
    S[j][2] = fast_exp2(S[j][2] - mn1); S[j][3] = fast_exp2(S[j][3] - mn1);
    s0 += S[j][0] + S[j][1];
    s1 += S[j][2] + S[j][3];
  }
  l[0] = l[0] * al0 + quad_sum(s0);
  l[1] = l[1] * al1 + quad_sum(s1);
#pragma unroll
  for (int n = 0; n < D / 8; ++n) { O[n][0] *= al0; O[n][1] *= al0; O[n][2] *= al1; O[n][3] *= al1; }
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    uint32_t a[4];
    a[0] = pack_bf16(S[2 * ks][0], S[2 * ks][1]);
    a[1] = pack_bf16(S[2 * ks][2], S[2 * ks][3]);
    a[2] = pack_bf16(S[2 * ks + 1][0], S[2 * ks + 1][1]);
    a[3] = pack_bf16(S[2 * ks + 1][2], S[2 * ks + 1][3]);
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sV + swz<CPR>(16 * ks + (lane & 7) + (((lane >> 3) & 1) << 3), 2 * np + (lane >> 4)),
                b0, b1, b2, b3);
      mma_bf16(O[2 * np], a, b0, b1);
      mma_bf16(O[2 * np + 1], a, b2, b3);
    }
  }
}

// Merge a block whose P was taken relative to its own row maxima (mb0, mb1):
// O = O*exp2(m - m') + f * vscale[c] * X, with f = exp2(mb - m') * pscale.
template <int D, typename XT>
__device__ __forceinline__ void merge_block(float (*O)[4], float* m, float* l, float mb0, float mb1,
                                            float lb0, float lb1, XT (*X)[4], float pscale,
                                            const float* vscale, int tq) {
  const float mn0 = fmaxf(m[0], mb0), mn1 = fmaxf(m[1], mb1);
  const float ao0 = fast_exp2(m[0] - mn0), ao1 = fast_exp2(m[1] - mn1);
  const float ab0 = fast_exp2(mb0 - mn0), ab1 = fast_exp2(mb1 - mn1);
  l[0] = l[0] * ao0 + lb0 * ab0;
  l[1] = l[1] * ao1 + lb1 * ab1;
  m[0] = mn0; m[1] = mn1;
  const float f0 = ab0 * pscale, f1 = ab1 * pscale;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const float v0 = vscale[8 * n + 2 * tq], v1 = vscale[8 * n + 2 * tq + 1];
    O[n][0] = O[n][0] * ao0 + f0 * v0 * (float)X[n][0];
    O[n][1] = O[n][1] * ao0 + f0 * v1 * (float)X[n][1];
    O[n][2] = O[n][2] * ao1 + f1 * v0 * (float)X[n][2];
    O[n][3] = O[n][3] * ao1 + f1 * v1 * (float)X[n][3];
  }
}

// Softmax numerators against the phase reference: p = exp2(s - r) (0 for a row
// with no reference yet); returns the row sums.
__device__ __forceinline__ void block_probs(float (*S)[4], float r0, float r1, float& lb0, float& lb1) {
  float s0 = 0.f, s1 = 0.f;
  const bool ok0 = r0 != -INFINITY, ok1 = r1 != -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    S[j][0] = ok0 ? fast_exp2(S[j][0] - r0) : 0.f; S[j][1] = ok0 ? fast_exp2(S[j][1] - r0) : 0.f;
    S[j][2] = ok1 ? fast_exp2(S[j][2] - r1) : 0.f; S[j][3] = ok1 ? fast_exp2(S[j][3] - r1) : 0.f;
    s0 += S[j][0] + S[j][1];
    s1 += S[j][2] + S[j][3];
  }
  lb0 = quad_sum(s0);
  lb1 = quad_sum(s1);
}

// INT8 scores of one key block (exact integers, as floats).
template <int D>
__device__ __forceinline__ void qk_int8(uint32_t sQ, uint32_t sK, int warp, int lane, float (*S)[4]) {
  constexpr int QCPR = D / 16;  // INT8 Q/K rows: D bytes
  int Si[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) Si[j][0] = Si[j][1] = Si[j][2] = Si[j][3] = 0;
#pragma unroll
  for (int kk = 0; kk < D / 32; ++kk) {
    uint32_t a[4];
    ldsm_x4(sQ + swz<QCPR>(warp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), 2 * kk + (lane >> 4)),
            a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sK + swz<QCPR>(16 * np + (lane & 7) + ((lane >> 4) << 3), 2 * kk + ((lane >> 3) & 1)),
              b0, b1, b2, b3);
      mma_s8s8(Si[2 * np], a, b0, b1);
      mma_s8s8(Si[2 * np + 1], a, b2, b3);
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) S[j][e] = (float)Si[j][e];
}

// One INT8 key block, P quantised against the phase reference r (2 rows).
template <int D>
__device__ __forceinline__ void block8(uint32_t sQ, uint32_t sK, uint32_t sV, uint8_t* sPw,
                                       unsigned long long vmask, float sc, int warp, int lane,
                                       float (*O)[4], float* m, float* l, const float* vscale,
                                       const float* r) {
  const int gq = lane >> 2, tq = lane & 3;
  float S[8][4];
  qk_int8<D>(sQ, sK, warp, lane, S);
  float mx0, mx1, lb0, lb1;
  scale_mask(S, sc, vmask, tq, mx0, mx1);
  block_probs(S, r[0], r[1], lb0, lb1);
  // u8 P codes, round(255 p), through this warp's [16][64] shared tile
  const uint32_t sP = smem_u32(sPw);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t c0 = __float2uint_rn(255.f * S[j][0]), c1 = __float2uint_rn(255.f * S[j][1]);
    const uint32_t c2 = __float2uint_rn(255.f * S[j][2]), c3 = __float2uint_rn(255.f * S[j][3]);
    const int inb = 8 * (j & 1) + 2 * tq;
    *reinterpret_cast<uint16_t*>(sPw + swz<4>(gq, j >> 1) + inb) = (uint16_t)(c0 | (c1 << 8));
    *reinterpret_cast<uint16_t*>(sPw + swz<4>(gq + 8, j >> 1) + inb) = (uint16_t)(c2 | (c3 << 8));
  }
  __syncwarp();
  int X[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) X[n][0] = X[n][1] = X[n][2] = X[n][3] = 0;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    uint32_t a[4];
    ldsm_x4(sP + swz<4>((lane & 7) + (((lane >> 3) & 1) << 3), 2 * ks + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sV + swz<4>(16 * np + (lane & 7) + ((lane >> 4) << 3), 2 * ks + ((lane >> 3) & 1)),
              b0, b1, b2, b3);
      mma_u8s8(X[2 * np], a, b0, b1);
      mma_u8s8(X[2 * np + 1], a, b2, b3);
    }
  }
  __syncwarp();
  merge_block<D, int>(O, m, l, r[0], r[1], lb0, lb1, X, 1.0f / 255.0f, vscale, tq);
}

// NVFP4 re-quantisation of 2688 p for 4 probabilities of one row's 16-key
// microblock (this lane's 4, the other 12 in the lane quad) → two f16x2
// A-fragment words holding the dequantised values (2688 p, quantised).
__device__ __forceinline__ void quant_p4(float p0, float p1, float p2, float p3, uint32_t& w01,
                                         uint32_t& w23) {
  p0 *= 2688.0f; p1 *= 2688.0f; p2 *= 2688.0f; p3 *= 2688.0f;
  float mx = fmaxf(fmaxf(p0, p1), fmaxf(p2, p3));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  const uint32_t sf = cvt_e4m3x2(0.f, __fdiv_rn(mx, 6.0f)) & 0xffu;
  const float dec = e4m3_to_f32(sf);
  if (dec == 0.f) { w01 = w23 = 0u; return; }
  const float r = __fdiv_rn(1.0f, dec);
  const __half2 d2 = __float2half2_rn(dec);
  uint32_t a = e2m1x2_to_f16x2(cvt_e2m1x2(__fmul_rn(p1, r), __fmul_rn(p0, r)));
  uint32_t b = e2m1x2_to_f16x2(cvt_e2m1x2(__fmul_rn(p3, r), __fmul_rn(p2, r)));
  __half2 ha = __hmul2(*reinterpret_cast<__half2*>(&a), d2);
  __half2 hb = __hmul2(*reinterpret_cast<__half2*>(&b), d2);
  w01 = *reinterpret_cast<uint32_t*>(&ha);
  w23 = *reinterpret_cast<uint32_t*>(&hb);
}

// One NVFP4 key block (K and V^T already dequantised to f16 in shared memory),
// P quantised against the phase reference r (2 rows).
template <int D>
__device__ __forceinline__ void block4(uint32_t sQ, uint32_t sK, uint32_t sVt, unsigned long long vmask,
                                       float sl2, int warp, int lane, float (*O)[4], float* m, float* l,
                                       const float* vscale, const float* r) {
  const int tq = lane & 3;
  float S[8][4];
  qk_16bit<D, true>(sQ, sK, warp, lane, S);
  float mx0, mx1, lb0, lb1;
  scale_mask(S, sl2, vmask, tq, mx0, mx1);
  block_probs(S, r[0], r[1], lb0, lb1);
  float X[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) X[n][0] = X[n][1] = X[n][2] = X[n][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    // keys 16ks.. : row gq holds S[2ks][0,1] and S[2ks+1][0,1]; row gq+8 the [2,3]s
    uint32_t a[4];
    quant_p4(S[2 * ks][0], S[2 * ks][1], S[2 * ks + 1][0], S[2 * ks + 1][1], a[0], a[2]);
    quant_p4(S[2 * ks][2], S[2 * ks][3], S[2 * ks + 1][2], S[2 * ks + 1][3], a[1], a[3]);
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sVt + swz<8>(16 * np + (lane & 7) + ((lane >> 4) << 3), 2 * ks + ((lane >> 3) & 1)),
              b0, b1, b2, b3);
      mma_f16(X[2 * np], a, b0, b1);
      mma_f16(X[2 * np + 1], a, b2, b3);
    }
  }
  merge_block<D, float>(O, m, l, r[0], r[1], lb0, lb1, X, 1.0f / 2688.0f, vscale, tq);
}

// Normalise, round to bf16, and write this warp's 16 rows to their tokens.
template <int D, typename TokFn>
__device__ __forceinline__ void store_rows(uint8_t* stile, __nv_bfloat16* out, float (*O)[4],
                                           const float* l, int warp, int lane, TokFn tok) {
  constexpr int CPR = D / 8;
  const int gq = lane >> 2, tq = lane & 3;
  const float i0 = l[0] > 0.f ? 1.f / l[0] : 0.f, i1 = l[1] > 0.f ? 1.f / l[1] : 0.f;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    *reinterpret_cast<uint32_t*>(stile + swz<CPR>(warp * 16 + gq, n) + 4 * tq) =
        pack_bf16(O[n][0] * i0, O[n][1] * i0);
    *reinterpret_cast<uint32_t*>(stile + swz<CPR>(warp * 16 + gq + 8, n) + 4 * tq) =
        pack_bf16(O[n][2] * i1, O[n][3] * i1);
  }
  __syncwarp();
  for (int e = lane; e < 16 * CPR; e += 32) {
    const int r = warp * 16 + e / CPR, c = e % CPR;
    const int t = tok(r);
    if (t >= 0)
      *reinterpret_cast<uint4*>(out + (size_t)t * D + c * 8) =
          *reinterpret_cast<const uint4*>(stile + swz<CPR>(r, c));
  }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 2) attn_mp_kernel(Geom g, AttnArgs A) {
  using SL = SmemLayout<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int qb = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row_lin = (size_t)bh * g.nb + qb;
  const int4 cnt = *reinterpret_cast<const int4*>(A.counts + row_lin * 4);
  const uint16_t* list = A.lists + row_lin * g.nb;
  const uint32_t s0 = smem_u32(smem);
  const float sl2 = kLog2e / sqrtf((float)D);
  float* vs = reinterpret_cast<float*>(smem + SL::VS);

  float O[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  const size_t head = (size_t)bh * g.N * D;
  auto qtok = [&](int r) { return slot_token(g, qb, r); };

  // ---------------- phase 16
  if (cnt.x > 0) {
    load_rows_bf16<D>(s0 + SL::Q, A.q + head, qtok);
    auto issue = [&](int j) {
      const int kb = list[j];
      auto ktok = [&](int r) { return slot_token(g, kb, r); };
      load_rows_bf16<D>(s0 + SL::K + (j & 1) * SL::TILE16, A.k + head, ktok);
      load_rows_bf16<D>(s0 + SL::V + (j & 1) * SL::TILE16, A.v + head, ktok);
      cp_async_commit();
    };
    issue(0);
    for (int j = 0; j < cnt.x; ++j) {
      if (j + 1 < cnt.x) { issue(j + 1); cp_async_wait<1>(); } else { cp_async_wait<0>(); }
      __syncthreads();
      block16<D>(s0 + SL::Q, s0 + SL::K + (j & 1) * SL::TILE16, s0 + SL::V + (j & 1) * SL::TILE16,
                 region_mask(g, list[j]), sl2, warp, lane, O, m, l);
      __syncthreads();
    }
  }
  // units of the low-bit phases: the pair's merged key lists, two entries at a
  // time; this query block takes the entries it is a member of
  const size_t prow = (size_t)bh * ((g.nb + 1) / 2) + (qb >> 1);
  const int4 pc = *reinterpret_cast<const int4*>(A.pcnt + prow * 4);
  const uint32_t* items = A.plist + prow * (size_t)(2 * g.nb);
  const int mbit = (qb & 1) ? 17 : 16;
  auto unit_members = [&](const uint32_t* it, int n, int i, int* kbs) {
    int nm = 0;
    for (int t = 0; t < 2 && i + t < n; ++t) {
      const uint32_t e = it[i + t];
      if ((e >> mbit) & 1u) kbs[nm++] = (int)(e & 0xffffu);
    }
    return nm;
  };
  // raise the phase reference to ceil(unit max) where the max exceeds it
  auto raise_ref = [&](float* r, float ux0, float ux1) {
    if (ux0 != -INFINITY && (r[0] == -INFINITY || ux0 > r[0])) r[0] = ceilf(ux0);
    if (ux1 != -INFINITY && (r[1] == -INFINITY || ux1 > r[1])) r[1] = ceilf(ux1);
  };
  const int tq = lane & 3;
  // the phases share the softmax statistics: the low-bit reference starts from
  // the 16-bit phase's, ceil of the running row maximum (-inf if it had no
  // block), and carries on from the 8-bit phase into the 4-bit one
  float r[2] = {m[0], m[1]};
  // ---------------- phase 8
  if (cnt.y > 0) {
    load_bytes_swz<D>(s0 + SL::Q, reinterpret_cast<const uint8_t*>(A.q_i8) + row_lin * 64 * D, 64);
    for (int c = threadIdx.x; c < D; c += kAttnThreads) vs[c] = A.v_s8[(size_t)bh * D + c];
    const float sq = A.q_s8[row_lin];
    const uint32_t* it8 = items + pc.x;
    for (int i = 0; i < pc.y; i += 2) {
      int kbs[2];
      const int nm = unit_members(it8, pc.y, i, kbs);
      if (nm == 0) continue;
      for (int t = 0; t < nm; ++t) {
        const size_t kl = (size_t)bh * g.nb + kbs[t];
        load_bytes_swz<D>(s0 + SL::K + t * SL::TILE16, reinterpret_cast<const uint8_t*>(A.k_i8) + kl * 64 * D, 64);
        load_bytes_swz<64>(s0 + SL::V + t * SL::TILE16, reinterpret_cast<const uint8_t*>(A.v_i8) + kl * 64 * D, D);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      float ux0 = -INFINITY, ux1 = -INFINITY;
      for (int t = 0; t < nm; ++t) {  // the unit's row maxima, scores only
        float S[8][4], mx0, mx1;
        qk_int8<D>(s0 + SL::Q, s0 + SL::K + t * SL::TILE16, warp, lane, S);
        scale_mask(S, sq * A.k_s8[(size_t)bh * g.nb + kbs[t]] * sl2, region_mask(g, kbs[t]), tq, mx0, mx1);
        ux0 = fmaxf(ux0, mx0); ux1 = fmaxf(ux1, mx1);
      }
      raise_ref(r, ux0, ux1);
      for (int t = 0; t < nm; ++t) {
        const float sc = sq * A.k_s8[(size_t)bh * g.nb + kbs[t]] * sl2;
        block8<D>(s0 + SL::Q, s0 + SL::K + t * SL::TILE16, s0 + SL::V + t * SL::TILE16,
                  smem + SL::P + warp * 1024, region_mask(g, kbs[t]), sc, warp, lane, O, m, l, vs, r);
      }
      __syncthreads();
    }
  }
  // ---------------- phase 4
  if (cnt.z > 0) {
    dequant_f4_tile<D>(smem + SL::Q, A.q_f4 + row_lin * 64 * (D / 2), A.q_sf4 + row_lin * SL::KSF, 64);
    for (int c = threadIdx.x; c < D; c += kAttnThreads) vs[c] = A.v_g4[(size_t)bh * D + c];
    const uint32_t* it4 = items + pc.x + pc.y;
    for (int i = 0; i < pc.z; i += 2) {
      int kbs[2];
      const int nm = unit_members(it4, pc.z, i, kbs);
      if (nm == 0) continue;
      for (int t = 0; t < nm; ++t) {
        const size_t kl = (size_t)bh * g.nb + kbs[t];
        const uint32_t raw = s0 + SL::RAW + t * SL::RAW_STAGE;
        load_bytes(raw + SL::RAW_KC, A.k_f4 + kl * 64 * (D / 2), 64 * D / 2);
        load_bytes(raw + SL::RAW_KS, A.k_sf4 + kl * SL::KSF, SL::KSF);
        load_bytes(raw + SL::RAW_VC, A.v_f4 + kl * D * 32, D * 32);
        load_bytes(raw + SL::RAW_VS, A.v_sf4 + kl * kSfAtomBytes, kSfAtomBytes);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      for (int t = 0; t < nm; ++t) {
        uint8_t* raw = smem + SL::RAW + t * SL::RAW_STAGE;
        dequant_f4_tile<D>(smem + SL::K + t * SL::TILE16, raw + SL::RAW_KC, raw + SL::RAW_KS, 64);
        dequant_f4_tile<64>(smem + SL::V + t * SL::TILE16, raw + SL::RAW_VC, raw + SL::RAW_VS, D);
      }
      __syncthreads();
      float ux0 = -INFINITY, ux1 = -INFINITY;
      for (int t = 0; t < nm; ++t) {  // the unit's row maxima, scores only
        float S[8][4], mx0, mx1;
        qk_16bit<D, true>(s0 + SL::Q, s0 + SL::K + t * SL::TILE16, warp, lane, S);
        scale_mask(S, sl2, region_mask(g, kbs[t]), tq, mx0, mx1);
        ux0 = fmaxf(ux0, mx0); ux1 = fmaxf(ux1, mx1);
      }
      raise_ref(r, ux0, ux1);
      for (int t = 0; t < nm; ++t)
        block4<D>(s0 + SL::Q, s0 + SL::K + t * SL::TILE16, s0 + SL::V + t * SL::TILE16, region_mask(g, kbs[t]),
                  sl2, warp, lane, O, m, l, vs, r);
      __syncthreads();
    }
  }
  store_rows<D>(smem + SL::Q, A.out + head, O, l, warp, lane, qtok);
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 2) attn_dense_kernel(int N, const __nv_bfloat16* q,
                                                                     const __nv_bfloat16* k,
                                                                     const __nv_bfloat16* v,
                                                                     __nv_bfloat16* out) {
  using SL = SmemLayout<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t s0 = smem_u32(smem);
  const float sl2 = kLog2e / sqrtf((float)D);
  const size_t head = (size_t)bh * N * D;
  float O[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  auto qtok = [&](int r) { const int t = qt * 64 + r; return t < N ? t : -1; };
  load_rows_bf16<D>(s0 + SL::Q, q + head, qtok);
  const int nkt = (N + 63) / 64;
  auto issue = [&](int j) {
    auto ktok = [&](int r) { const int t = j * 64 + r; return t < N ? t : -1; };
    load_rows_bf16<D>(s0 + SL::K + (j & 1) * SL::TILE16, k + head, ktok);
    load_rows_bf16<D>(s0 + SL::V + (j & 1) * SL::TILE16, v + head, ktok);
    cp_async_commit();
  };
  issue(0);
  for (int j = 0; j < nkt; ++j) {
    if (j + 1 < nkt) { issue(j + 1); cp_async_wait<1>(); } else { cp_async_wait<0>(); }
    __syncthreads();
    const int rem = N - j * 64;
    const unsigned long long vmask = rem >= 64 ? ~0ull : ((1ull << rem) - 1ull);
    block16<D>(s0 + SL::Q, s0 + SL::K + (j & 1) * SL::TILE16, s0 + SL::V + (j & 1) * SL::TILE16,
               vmask, sl2, warp, lane, O, m, l);
    __syncthreads();
  }
  store_rows<D>(smem + SL::Q, out + head, O, l, warp, lane, qtok);
}

template <int D>
AttnArgs make_args(const Layout& L, const void* q, const void* k, const void* v, void* ws, void* out) {
  AttnArgs A;
  A.q = static_cast<const __nv_bfloat16*>(q);
  A.k = static_cast<const __nv_bfloat16*>(k);
  A.v = static_cast<const __nv_bfloat16*>(v);
  A.out = static_cast<__nv_bfloat16*>(out);
  A.q_i8 = at<int8_t>(ws, L, R_Q_I8); A.k_i8 = at<int8_t>(ws, L, R_K_I8); A.v_i8 = at<int8_t>(ws, L, R_V_I8);
  A.q_s8 = at<float>(ws, L, R_Q_S8); A.k_s8 = at<float>(ws, L, R_K_S8); A.v_s8 = at<float>(ws, L, R_V_S8);
  A.q_f4 = at<uint8_t>(ws, L, R_Q_F4); A.k_f4 = at<uint8_t>(ws, L, R_K_F4);
  A.q_sf4 = at<uint8_t>(ws, L, R_Q_SF4); A.k_sf4 = at<uint8_t>(ws, L, R_K_SF4);
  A.v_f4 = at<uint8_t>(ws, L, R_V_F4); A.v_sf4 = at<uint8_t>(ws, L, R_V_SF4);
  A.v_g4 = at<float>(ws, L, R_V_G4);
  A.lists = at<uint16_t>(ws, L, R_LISTS);
  A.counts = at<int>(ws, L, R_COUNTS);
  A.plist = at<uint32_t>(ws, L, R_PLIST);
  A.pcnt = at<int>(ws, L, R_PCNT);
  return A;
}

template <int D>
cudaError_t launch_attention_d(const Geom& g, const Layout& L, const void* q, const void* k,
                               const void* v, void* ws, void* out, cudaStream_t st) {
  const int smem = SmemLayout<D>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(attn_mp_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if ((e = launch_pair_lists(g, L, ws, st)) != cudaSuccess) return e;
  attn_mp_kernel<D><<<dim3(g.nb, g.BH), kAttnThreads, smem, st>>>(g, make_args<D>(L, q, k, v, ws, out));
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_dense_d(int B, int H, int N, const void* q, const void* k, const void* v, void* out,
                           cudaStream_t st) {
  const int smem = SmemLayout<D>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(attn_dense_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_dense_kernel<D><<<dim3((N + 63) / 64, B * H), kAttnThreads, smem, st>>>(
      N, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Geom& g, const Layout& L, const void* q, const void* k, const void* v,
                             void* ws, void* out, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(at<int>(ws, L, R_STATUS), 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  if (attention_tc_supported(g)) return launch_attention_tc(g, L, q, k, v, ws, out, st);
  return g.d == 128 ? launch_attention_d<128>(g, L, q, k, v, ws, out, st)
                    : launch_attention_d<64>(g, L, q, k, v, ws, out, st);
}

cudaError_t launch_dense(int B, int H, int N, int d, const void* q, const void* k, const void* v, void* out,
                         cudaStream_t st) {
  if (dense_tc_supported(B, H, N, d)) return launch_dense_tc(B, H, N, q, k, v, out, st);
  return d == 128 ? launch_dense_d<128>(B, H, N, q, k, v, out, st)
                  : launch_dense_d<64>(B, H, N, q, k, v, out, st);
}

}  // namespace da2
