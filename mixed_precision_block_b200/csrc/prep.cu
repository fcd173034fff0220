// Stage 1: fused operand preparation.
//
// DraftAttention2 abstract and reading note (Method overview bullet 4,
// Figure 3(b)): Q/K reordering, pooling and quantisation share one kernel;
// V is reordered and transposed while it is packed.
//
// prep_qk_tma: persistent; each CTA walks (tensor Q|K, head, region block)
//   items, one thread keeping a ring of region tiles in flight with TMA (an
//   8x8-token box per 64 channels straight from the [B,H,N,d] input, zero
//   outside the frame).  From shared memory the CTA produces the pooled mean /
//   max (warp-shuffle + shared-memory reductions), the INT8 codes with the
//   block's absmax scale, and the NVFP4 codes with one e4m3 scale per 16
//   channels of a token.
// v_amax + pack_v_tma: the per-channel absmax of V over all real tokens of a
//   head (first pass, atomicMax on the float bits), then the same TMA ring
//   over V's region tiles, which writes INT8 and NVFP4 codes in
//   [block][channel][token] order.
#include "da2_internal.cuh"
#include "sm100.cuh"

namespace da2 {
namespace {

constexpr int kThreads = 256;

struct PrepPtrs {
  const __nv_bfloat16* x[2];
  float* avg[2];
  float* mx[2];
  int8_t* i8[2];
  float* s8[2];
  uint8_t* f4[2];
  uint8_t* sf4[2];
  int* perm;
};

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// NVFP4 microblock of 16 values held as 8 per lane in lanes (2j, 2j+1):
// returns 4 code bytes for this lane's 8 values and the e4m3 scale byte.
__device__ __forceinline__ uint32_t quant_f4x8(const float* x, float amax16, uint32_t* sf_byte) {
  const float t = __fdiv_rn(amax16, 6.0f);
  const uint32_t sf = cvt_e4m3x2(0.0f, t) & 0xffu;
  *sf_byte = sf;
  const float dec = e4m3_to_f32(sf);
  if (dec == 0.0f) return 0u;
  const float r = __fdiv_rn(1.0f, dec);
  uint32_t out = 0;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint32_t b = cvt_e2m1x2(__fmul_rn(x[2 * m + 1], r), __fmul_rn(x[2 * m], r));
    out |= b << (8 * m);
  }
  return out;
}

// bytes 0 of four words -> one word (x0 in the low byte)
__device__ __forceinline__ uint32_t low_bytes4(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3) {
  uint32_t lo, hi, r;
  asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(lo) : "r"(x0), "r"(x1));
  asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(hi) : "r"(x2), "r"(x3));
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(r) : "r"(lo), "r"(hi));
  return r;
}

// prep_qk_tma: persistent form of prep_qk.  Each CTA walks work items
// (tensor, head, region block) with stride gridDim.x; one thread keeps a ring
// of kPrepStages region tiles in flight with TMA (a {64 ch, rw, rh, 1} box per
// 64 channels: the 8x8 region straight from the [B,H,N,d] tensor, zero outside
// the frame), and the CTA computes from shared memory what prep_qk computes
// from registers.
constexpr int kPrepStages = 4;

template <int D>
struct PrepTmaLayout {
  static constexpr int BOX = 64 * 64 * 2;  // one 64-channel region box, bf16
  static constexpr int STAGE = (D / 64) * BOX;
  static constexpr int SUM = kPrepStages * STAGE;            // float [8 warps][D]
  static constexpr int MAX = SUM + 8 * D * 4;                // float [8 warps][D]
  static constexpr int AMAX = MAX + 8 * D * 4;               // float [8]
  static constexpr int BAR = AMAX + 64;                      // mbarriers [kPrepStages]
  static constexpr int INFO = BAR + 8 * kPrepStages;         // int4 [kPrepStages]: item, blk, vy, vx
  static constexpr int TOTAL = INFO + 16 * kPrepStages;
};

template <int D>
__global__ void __launch_bounds__(kThreads) prep_qk_tma_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                               const __grid_constant__ CUtensorMap tmK, Geom g,
                                                               PrepPtrs P, int want_i8, int want_f4, int n_items) {
  using LY = PrepTmaLayout<D>;
  constexpr int CPT = D / 8;                // 16-byte chunks per token
  constexpr int NC = 64 * CPT / kThreads;   // chunks per thread
  constexpr int SLOT_STEP = kThreads / CPT;
  extern __shared__ __align__(1024) uint8_t psm[];
  const uint32_t s0 = (uint32_t)__cvta_generic_to_shared(psm);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = tid % CPT, slot0 = tid / CPT;
  float* s_sum = reinterpret_cast<float*>(psm + LY::SUM);
  float* s_max = reinterpret_cast<float*>(psm + LY::MAX);
  float* s_amax = reinterpret_cast<float*>(psm + LY::AMAX);
  auto bar = [&](int i) { return s0 + LY::BAR + 8u * (uint32_t)i; };
  const int t_of = g.nry * g.nrx;
  int4* info = reinterpret_cast<int4*>(psm + LY::INFO);
  const int lrw = __ffs(g.rw) - 1;  // region width is a power of two (rw * rh = 64)
  // item -> (tensor, head, block), decoded once by the issuing thread and
  // published with the stage; the TMA load of one item into a stage
  auto issue = [&](int item, int stage) {
    const int rest = item >> 1;
    const int bh = rest / g.nb, blk = rest - bh * g.nb;
    const int t = blk / t_of, rem = blk - t * t_of;
    const int ry = rem / g.nrx, rx = rem - ry * g.nrx;
    info[stage] = make_int4(item, blk, min(g.rh, g.Hh - ry * g.rh), min(g.rw, g.Ww - rx * g.rw));
    const int which = item & 1;
    const uint32_t fb = bar(stage);
    sm100::mbar_expect_tx(fb, (uint32_t)LY::STAGE);
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      sm100::tma_load_4d(s0 + stage * LY::STAGE + c * LY::BOX, which ? &tmK : &tmQ, fb, 64 * c, rx * g.rw,
                         ry * g.rh, bh * g.T + t);
  };
  if (tid == 0) {
    for (int s = 0; s < kPrepStages; ++s) sm100::mbar_init(bar(s), 1);
    sm100::fence_mbar_init();
    sm100::prefetch_tmap(&tmQ);
    sm100::prefetch_tmap(&tmK);
    for (int s = 0; s < kPrepStages; ++s) {
      const int item = blockIdx.x + s * gridDim.x;
      if (item < n_items) issue(item, s);
    }
  }
  __syncthreads();
  for (int k = 0;; ++k) {
    const int item = blockIdx.x + k * gridDim.x;
    if (item >= n_items) break;
    const int stage = k % kPrepStages;
    // bounded wait, agreed by the whole CTA so that no thread leaves alone
    if (!__syncthreads_and(sm100::mbar_wait(bar(stage), (uint32_t)(k / kPrepStages) & 1u))) break;
    const int4 inf = info[stage];  // written before the stage's TMA was issued
    const int which = item & 1, blk = inf.y, vy = inf.z, vx = inf.w;
    const int bh = (item >> 1) / g.nb;
    const uint8_t* tile = psm + stage * LY::STAGE;
    float v[NC][8];
    bool valid[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int s = slot0 + i * SLOT_STEP;
      valid[i] = (s >> lrw) < vy && (s & (g.rw - 1)) < vx;
      const uint4 u = *reinterpret_cast<const uint4*>(tile + (cg >> 3) * LY::BOX + s * 128 + (cg & 7) * 16);
      unpack8(u, v[i]);
    }
    __syncthreads();  // every thread has its values: the stage may be refilled
    if (tid == 0) {
      const int nxt = blockIdx.x + (k + kPrepStages) * gridDim.x;
      if (nxt < n_items) issue(nxt, stage);
    }
    if (which == 0 && bh == 0 && tid < 64) P.perm[blk * 64 + tid] = slot_token(g, blk, tid);
    // ---- pooled mean and max over real tokens; absmax over the block
    float psum[8], pmax[8], amax = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) { psum[c] = 0.f; pmax[c] = -INFINITY; }
#pragma unroll
    for (int i = 0; i < NC; ++i) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (valid[i]) { psum[c] += v[i][c]; pmax[c] = fmaxf(pmax[c], v[i][c]); }
        amax = fmaxf(amax, fabsf(v[i][c]));  // padding slots hold the TMA zero fill
      }
    }
#pragma unroll
    for (int o = CPT; o < 32; o <<= 1) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        psum[c] += __shfl_xor_sync(0xffffffffu, psum[c], o);
        pmax[c] = fmaxf(pmax[c], __shfl_xor_sync(0xffffffffu, pmax[c], o));
      }
    }
    if (lane < CPT) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        s_sum[warp * D + cg * 8 + c] = psum[c];
        s_max[warp * D + cg * 8 + c] = pmax[c];
      }
    }
    amax = warp_max(amax);
    if (lane == 0) s_amax[warp] = amax;
    __syncthreads();
    const size_t blk_lin = (size_t)bh * g.nb + blk;
    if (tid < D) {
      float s = 0.f, m = -INFINITY;
#pragma unroll
      for (int w = 0; w < kThreads / 32; ++w) { s += s_sum[w * D + tid]; m = fmaxf(m, s_max[w * D + tid]); }
      (which ? P.avg[1] : P.avg[0])[blk_lin * D + tid] = s / (float)(vy * vx);
      (which ? P.mx[1] : P.mx[0])[blk_lin * D + tid] = m;
    }
    amax = s_amax[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, s_amax[w]);
    // ---- INT8: one symmetric scale per block; rint through the mantissa of
    // 1.5*2^23 (|x * 127/amax| <= 127 needs no clamp), the code in the low byte
    if (want_i8) {
      const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
      if (tid == 0) (which ? P.s8[1] : P.s8[0])[blk_lin] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.f;
      int8_t* __restrict__ dst = (which ? P.i8[1] : P.i8[0]) + blk_lin * 64 * D;
#pragma unroll
      for (int i = 0; i < NC; ++i) {
        const int s = slot0 + i * SLOT_STEP;
        uint32_t c[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) c[e] = __float_as_uint(__fadd_rn(__fmul_rn(v[i][e], inv), 12582912.0f));
        uint2 w;
        w.x = low_bytes4(c[0], c[1], c[2], c[3]);
        w.y = low_bytes4(c[4], c[5], c[6], c[7]);
        *reinterpret_cast<uint2*>(dst + (size_t)s * D + cg * 8) = w;
      }
    }
    // ---- NVFP4: e4m3 scale per 16 channels of a token
    if (want_f4) {
      uint8_t* __restrict__ dst = (which ? P.f4[1] : P.f4[0]) + blk_lin * 64 * (D / 2);
      uint8_t* __restrict__ sfd = (which ? P.sf4[1] : P.sf4[0]) + blk_lin * (D / 64) * kSfAtomBytes;
#pragma unroll
      for (int i = 0; i < NC; ++i) {
        const int s = slot0 + i * SLOT_STEP;
        float a8 = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) a8 = fmaxf(a8, fabsf(v[i][c]));
        const float a16 = fmaxf(a8, __shfl_xor_sync(0xffffffffu, a8, 1));
        uint32_t sfb;
        const uint32_t codes = quant_f4x8(v[i], a16, &sfb);
        *reinterpret_cast<uint32_t*>(dst + (size_t)s * (D / 2) + cg * 4) = codes;
        if ((cg & 1) == 0) {
          const int o = sf_atom_offset(s, cg / 2);
          sfd[o] = (uint8_t)sfb;
          sfd[o + 8] = (uint8_t)sfb;  // rows 64..127 of the atom repeat rows 0..63
        }
      }
    }
  }
}

// Per-channel absmax of V over all real tokens of one head.
template <int D>
__global__ void __launch_bounds__(kThreads) v_amax_kernel(Geom g, const __nv_bfloat16* __restrict__ v,
                                                          unsigned int* __restrict__ amax_bits,
                                                          int tokens_per_cta) {
  constexpr int CPT = D / 8;
  constexpr int ROWS = kThreads / CPT;
  const int bh = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = tid % CPT;
  const int t0 = blockIdx.x * tokens_per_cta;
  const int t1 = min(g.N, t0 + tokens_per_cta);
  const __nv_bfloat16* __restrict__ x = v + (size_t)bh * g.N * D;
  float m[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) m[c] = 0.f;
  for (int t = t0 + tid / CPT; t < t1; t += ROWS) {
    float f[8];
    unpack8(*reinterpret_cast<const uint4*>(x + (size_t)t * D + cg * 8), f);
#pragma unroll
    for (int c = 0; c < 8; ++c) m[c] = fmaxf(m[c], fabsf(f[c]));
  }
#pragma unroll
  for (int o = CPT; o < 32; o <<= 1)
#pragma unroll
    for (int c = 0; c < 8; ++c) m[c] = fmaxf(m[c], __shfl_xor_sync(0xffffffffu, m[c], o));
  __shared__ float s_m[kThreads / 32][D];
  if (lane < CPT)
#pragma unroll
    for (int c = 0; c < 8; ++c) s_m[warp][cg * 8 + c] = m[c];
  __syncthreads();
  if (tid < D) {
    float r = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) r = fmaxf(r, s_m[w][tid]);
    atomicMax(amax_bits + (size_t)bh * D + tid, __float_as_uint(r));  // r >= 0: bit order = value order
  }
}

struct VPtrs {
  const __nv_bfloat16* v;
  const unsigned int* amax_bits;
  __nv_bfloat16* q8;  // INT8 codes as bf16 values, [block][slot][channel]
  float* s8;
  uint8_t* f4;
  uint8_t* sf4;
  float* g4;
};

// pack_v_tma: persistent form of pack_v with the same TMA ring as
// prep_qk_tma.  The tile stays as loaded ([slot][channel], bf16); a thread
// takes two neighbouring channels of one 16-slot group, reads them down the
// slots (a warp covers 64 channels: conflict-free) and writes both channels'
// INT8 codes and NVFP4 microblock in [block][channel][slot] order.
template <int D>
__global__ void __launch_bounds__(kThreads) pack_v_tma_kernel(const __grid_constant__ CUtensorMap tmV, Geom g,
                                                              VPtrs P, int want_i8, int want_f4, int n_items) {
  using LY = PrepTmaLayout<D>;
  static_assert(D / 2 * 4 == kThreads || D / 2 * 4 == kThreads / 2, "one or half a unit per thread");
  constexpr int UNITS = D / 2 * 4;  // (channel pair, 16-slot group)
  extern __shared__ __align__(1024) uint8_t psm[];
  const uint32_t s0 = (uint32_t)__cvta_generic_to_shared(psm);
  const int tid = threadIdx.x;
  auto bar = [&](int i) { return s0 + LY::BAR + 8u * (uint32_t)i; };
  int4* info = reinterpret_cast<int4*>(psm + LY::INFO);
  const int t_of = g.nry * g.nrx;
  auto issue = [&](int item, int stage) {
    const int bh = item / g.nb, blk = item - bh * g.nb;
    const int t = blk / t_of, rem = blk - t * t_of;
    const int ry = rem / g.nrx, rx = rem - ry * g.nrx;
    info[stage] = make_int4(bh, blk, 0, 0);
    const uint32_t fb = bar(stage);
    sm100::mbar_expect_tx(fb, (uint32_t)LY::STAGE);
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      sm100::tma_load_4d(s0 + stage * LY::STAGE + c * LY::BOX, &tmV, fb, 64 * c, rx * g.rw, ry * g.rh, bh * g.T + t);
  };
  if (tid == 0) {
    for (int s = 0; s < kPrepStages; ++s) sm100::mbar_init(bar(s), 1);
    sm100::fence_mbar_init();
    sm100::prefetch_tmap(&tmV);
    for (int s = 0; s < kPrepStages; ++s) {
      const int item = blockIdx.x + s * gridDim.x;
      if (item < n_items) issue(item, s);
    }
  }
  __syncthreads();
  const int cp = tid % (D / 2), j = tid / (D / 2);  // channel pair, 16-slot group
  const int c0 = 2 * cp;
  const bool active = tid < UNITS;
  for (int k = 0;; ++k) {
    const int item = blockIdx.x + k * gridDim.x;
    if (item >= n_items) break;
    const int stage = k % kPrepStages;
    // bounded wait, agreed by the whole CTA so that no thread leaves alone
    if (!__syncthreads_and(sm100::mbar_wait(bar(stage), (uint32_t)(k / kPrepStages) & 1u))) break;
    const int4 inf = info[stage];
    const int bh = inf.x, blk = inf.y;
    const size_t blk_lin = (size_t)bh * g.nb + blk;
    float f0[16], f1[16];
    if (active) {
      const uint8_t* col = psm + stage * LY::STAGE + (c0 >> 6) * LY::BOX + (c0 & 63) * 2;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float2 t2 = __bfloat1622float2(
            *reinterpret_cast<const __nv_bfloat162*>(col + (16 * j + e) * 128));
        f0[e] = t2.x;
        f1[e] = t2.y;
      }
    }
    __syncthreads();  // every thread has its values: the stage may be refilled
    if (tid == 0) {
      const int nxt = blockIdx.x + (k + kPrepStages) * gridDim.x;
      if (nxt < n_items) issue(nxt, stage);
    }
    const unsigned int* amax_bits = P.amax_bits + (size_t)bh * D;
    if (blk == 0 && tid < D) {
      const float a = __uint_as_float(amax_bits[tid]);
      if (want_i8) P.s8[(size_t)bh * D + tid] = a > 0.f ? __fdiv_rn(a, 127.0f) : 0.f;
      if (want_f4) P.g4[(size_t)bh * D + tid] = __fdiv_rn(a, 2688.0f);
    }
    if (!active) continue;
    if (want_i8) {
      // the codes of channels c0, c0+1 for this thread's 16 slots, as bf16
      // values (integers up to 127: exact), in the block's [slot][channel]
      // order — the layout of a bf16 V tile, so the INT8 phase's P·V runs on
      // the same tensor-core path as the 16-bit phase's
      const float a0 = __uint_as_float(amax_bits[c0]), a1 = __uint_as_float(amax_bits[c0 + 1]);
      const float inv0 = a0 > 0.f ? __fdiv_rn(127.0f, a0) : 0.f, inv1 = a1 > 0.f ? __fdiv_rn(127.0f, a1) : 0.f;
      __nv_bfloat16* dst = P.q8 + (blk_lin * 64 + 16 * j) * D + c0;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int k0 = max(-127, min(127, __float2int_rn(__fmul_rn(f0[e], inv0))));
        const int k1 = max(-127, min(127, __float2int_rn(__fmul_rn(f1[e], inv1))));
        *reinterpret_cast<__nv_bfloat162*>(dst + (size_t)e * D) =
            __floats2bfloat162_rn((float)k0, (float)k1);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float* f = h ? f1 : f0;
      const int c = c0 + h;
      const float a = __uint_as_float(amax_bits[c]);
      if (want_f4) {
        const float gch = __fdiv_rn(a, 2688.0f);
        const float r = gch > 0.f ? __fdiv_rn(1.0f, gch) : 0.f;
        float a16 = 0.f;
        float y[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) { y[e] = __fmul_rn(f[e], r); a16 = fmaxf(a16, fabsf(y[e])); }
        uint32_t sfb;
        uint2 w;
        w.x = quant_f4x8(y, a16, &sfb);
        w.y = quant_f4x8(y + 8, a16, &sfb);
        *reinterpret_cast<uint2*>(P.f4 + (blk_lin * D + c) * 32 + 8 * j) = w;
        P.sf4[blk_lin * kSfAtomBytes + sf_atom_offset(c, j)] = (uint8_t)sfb;
      }
    }
  }
}

template <int D>
cudaError_t launch_prepare_d(const Geom& g, const Layout& L, const void* q, const void* k,
                             const void* v, void* ws, cudaStream_t st) {
  const int want_i8 = g.n8 > 0, want_f4 = g.n4 > 0;
  PrepPtrs P;
  P.x[0] = static_cast<const __nv_bfloat16*>(q);
  P.x[1] = static_cast<const __nv_bfloat16*>(k);
  P.avg[0] = at<float>(ws, L, R_Q_AVG); P.avg[1] = at<float>(ws, L, R_K_AVG);
  P.mx[0] = at<float>(ws, L, R_Q_MAX); P.mx[1] = at<float>(ws, L, R_K_MAX);
  P.i8[0] = at<int8_t>(ws, L, R_Q_I8); P.i8[1] = at<int8_t>(ws, L, R_K_I8);
  P.s8[0] = at<float>(ws, L, R_Q_S8); P.s8[1] = at<float>(ws, L, R_K_S8);
  P.f4[0] = at<uint8_t>(ws, L, R_Q_F4); P.f4[1] = at<uint8_t>(ws, L, R_K_F4);
  P.sf4[0] = at<uint8_t>(ws, L, R_Q_SF4); P.sf4[1] = at<uint8_t>(ws, L, R_K_SF4);
  P.perm = at<int>(ws, L, R_PERM);
  cudaError_t e;
  CUtensorMap tq, tk;
  if (make_region_map(&tq, q, g, false) && make_region_map(&tk, k, g, false)) {
    using LY = PrepTmaLayout<D>;
    e = cudaFuncSetAttribute(prep_qk_tma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::TOTAL);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prep_qk_tma_kernel<D>, kThreads, LY::TOTAL);
    const int n_items = 2 * g.BH * g.nb;
    const int grid = std::max(1, std::min(n_items, sms * std::max(per_sm, 1)));
    prep_qk_tma_kernel<D><<<grid, kThreads, LY::TOTAL, st>>>(tq, tk, g, P, want_i8, want_f4, n_items);
  } else {
    return cudaErrorNotSupported;  // no tensor-map encoder in this driver
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || !(want_i8 || want_f4)) return e;

  unsigned int* amax = at<unsigned int>(ws, L, R_V_AMAX);
  e = cudaMemsetAsync(amax, 0, L.size[R_V_AMAX], st);
  if (e != cudaSuccess) return e;
  const int tpc = 2048;
  v_amax_kernel<D><<<dim3((g.N + tpc - 1) / tpc, g.BH), kThreads, 0, st>>>(
      g, static_cast<const __nv_bfloat16*>(v), amax, tpc);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  VPtrs V{static_cast<const __nv_bfloat16*>(v), amax, at<__nv_bfloat16>(ws, L, R_V_I8),
          at<float>(ws, L, R_V_S8), at<uint8_t>(ws, L, R_V_F4), at<uint8_t>(ws, L, R_V_SF4),
          at<float>(ws, L, R_V_G4)};
  CUtensorMap tv;
  if (make_region_map(&tv, v, g, false)) {
    using LY = PrepTmaLayout<D>;
    e = cudaFuncSetAttribute(pack_v_tma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::TOTAL);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pack_v_tma_kernel<D>, kThreads, LY::TOTAL);
    const int n_items = g.BH * g.nb;
    const int grid = std::max(1, std::min(n_items, sms * std::max(per_sm, 1)));
    pack_v_tma_kernel<D><<<grid, kThreads, LY::TOTAL, st>>>(tv, g, V, want_i8, want_f4, n_items);
  } else {
    return cudaErrorNotSupported;  // no tensor-map encoder in this driver
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prepare(const Geom& g, const Layout& L, const void* q, const void* k,
                           const void* v, void* ws, cudaStream_t st) {
  return g.d == 128 ? launch_prepare_d<128>(g, L, q, k, v, ws, st)
                    : launch_prepare_d<64>(g, L, q, k, v, ws, st);
}

}  // namespace da2
