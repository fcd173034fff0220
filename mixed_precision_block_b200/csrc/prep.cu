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
// v_prep: V's per-channel absmax over all real tokens of a head (atomicMax
//   on the float bits) and, once a head's absmax is complete, the same TMA ring
//   over V's region tiles writing the INT8 and NVFP4 codes — one persistent
//   kernel that orders its work so that V crosses HBM once (see v_prep_kernel).
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
constexpr uint32_t kPrepSpin = 1u << 22;  // bound of every wait (polls)

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

struct VPtrs {
  const __nv_bfloat16* v;
  unsigned int* amax_bits;  // per head and channel: absmax float bits (merged by atomicMax)
  __nv_bfloat16* q8;  // INT8 codes as bf16 values, [block][slot][channel]
  float* s8;
  uint8_t* f4;
  uint8_t* sf4;
  float* g4;
};

__device__ __forceinline__ unsigned int ld_acquire(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// v_prep: V in one pass over HBM.  A head's INT8 and NVFP4 channel scales need
// the absmax of every channel over all of the head's tokens before any code is
// written.  So the persistent CTAs take work items from a global counter in
// the order A(0), B(0), A(1), B(1), ..., where A(h) and B(h) hold one item per
// V block of head h.  An A(h) item takes the
// block's channel absmax into the CTA's running absmax of head h, which the
// CTA merges into the head's (atomicMax on the float bits) and counts as done
// when it moves to another head's A items, runs out of items, or is about to
// wait for a head h' >= h.  A B(h) item writes the block's codes once all of
// head h's A items are counted (a bounded wait: the CTAs still on head h's
// last A items).  Head h's V tiles were read just before and are still in L2
// (126 MB against 30 MB per head), so DRAM sees V once.  (Handing out A(h+1)
// between A(h) and B(h), to hide that wait, let a third of V drop out of L2.)
// The waits end, by induction on the head: an A item never waits, so a CTA
// holding unmerged A(h) items waits only for heads before h, which end by the
// induction; it then reaches its next A head, B(h' >= h) or the end of the
// items, and merges.  (Keeping A(h) unmerged while waiting for a later head
// can deadlock: that head's A items may sit behind waits for head h.)  The tile stays as loaded ([slot][channel],
// bf16); a thread takes two neighbouring channels of one 16-slot group, reads
// them down the slots (a warp covers 64 channels: conflict-free).
template <int D>
__global__ void __launch_bounds__(kThreads) v_prep_kernel(const __grid_constant__ CUtensorMap tmV, Geom g, VPtrs P,
                                                          int want_i8, int want_f4, int n_items,
                                                          unsigned int* __restrict__ work,
                                                          unsigned int* __restrict__ done, int* __restrict__ status,
                                                          uint32_t spin) {
  using LY = PrepTmaLayout<D>;
  static_assert(D / 2 * 4 == kThreads || D / 2 * 4 == kThreads / 2, "one or half a unit per thread");
  constexpr int UNITS = D / 2 * 4;  // (channel pair, 16-slot group)
  extern __shared__ __align__(1024) uint8_t psm[];
  const uint32_t s0 = (uint32_t)__cvta_generic_to_shared(psm);
  const int tid = threadIdx.x;
  auto bar = [&](int i) { return s0 + LY::BAR + 8u * (uint32_t)i; };
  int4* info = reinterpret_cast<int4*>(psm + LY::INFO);
  float* s_red = reinterpret_cast<float*>(psm + LY::SUM);       // [4 slot groups][D] absmax partials
  volatile int* s_go = reinterpret_cast<volatile int*>(psm + LY::AMAX);
  const int t_of = g.nry * g.nrx;
  // item -> (pack, head, block) in the order A(0), B(0), A(1), B(1), ...
  auto decode = [&](int item, int& is_b, int& bh, int& blk) {
    const int grp = item / g.nb;
    blk = item - grp * g.nb;
    bh = grp >> 1;
    is_b = grp & 1;
  };
  // this CTA's running absmax of head acc_bh over acc_n A items, not yet merged
  float* s_acc = reinterpret_cast<float*>(psm + LY::MAX);
  int acc_bh = -1, acc_n = 0;
  auto flush = [&]() {
    if (acc_n == 0) return;
    if (tid < D) {
      atomicMax(P.amax_bits + (size_t)acc_bh * D + tid, __float_as_uint(s_acc[tid]));  // >= 0: bit order = value order
      __threadfence();
    }
    __syncthreads();  // the merges are visible before the items count as done
    if (tid == 0) atomicAdd(done + acc_bh, (unsigned int)acc_n);
    acc_n = 0;
    acc_bh = -1;
  };
  // the issuing thread takes the next item and loads its V tile into `stage`,
  // or marks the stage empty once the items are exhausted
  auto issue = [&](int stage) {
    const int item = (int)atomicAdd(work, 1u);
    const uint32_t fb = bar(stage);
    if (item >= n_items) {
      info[stage] = make_int4(-1, 0, 0, 0);
      sm100::mbar_arrive(fb);
      return;
    }
    int is_b, bh, blk;
    decode(item, is_b, bh, blk);
    const int t = blk / t_of, rem = blk - t * t_of;
    const int ry = rem / g.nrx, rx = rem - ry * g.nrx;
    info[stage] = make_int4(is_b, bh, blk, 0);
    sm100::mbar_expect_tx(fb, (uint32_t)LY::STAGE);
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      sm100::tma_load_4d(s0 + stage * LY::STAGE + c * LY::BOX, &tmV, fb, 64 * c, rx * g.rw, ry * g.rh, bh * g.T + t);
  };
  if (tid == 0) {
    for (int s = 0; s < kPrepStages; ++s) sm100::mbar_init(bar(s), 1);
    sm100::fence_mbar_init();
    sm100::prefetch_tmap(&tmV);
    for (int s = 0; s < kPrepStages; ++s) issue(s);
  }
  __syncthreads();
  const int cp = tid % (D / 2), j = tid / (D / 2);  // channel pair, 16-slot group
  const int c0 = 2 * cp;
  const bool active = tid < UNITS;
  for (int k = 0;; ++k) {
    const int stage = k % kPrepStages;
    // bounded wait, agreed by the whole CTA so that no thread leaves alone
    if (!__syncthreads_and(sm100::mbar_wait(bar(stage), (uint32_t)(k / kPrepStages) & 1u, spin))) {
      if (tid == 0) atomicOr(status, 1);
      break;
    }
    const int4 inf = info[stage];
    // items are taken in increasing order, so the first empty stage comes after every loaded one
    if (inf.x < 0) break;
    const int is_b = inf.x, bh = inf.y, blk = inf.z;
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
    if (tid == 0) issue(stage);
    if (!is_b) {
      // ---- A: the block's channel absmax (padding slots hold the TMA zero fill) into the CTA's running one
      if (acc_bh != bh) flush();
      if (active) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) { a0 = fmaxf(a0, fabsf(f0[e])); a1 = fmaxf(a1, fabsf(f1[e])); }
        s_red[j * D + c0] = a0;
        s_red[j * D + c0 + 1] = a1;
      }
      __syncthreads();
      if (tid < D) {
        float r = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) r = fmaxf(r, s_red[q * D + tid]);
        s_acc[tid] = acc_n == 0 ? r : fmaxf(s_acc[tid], r);
      }
      acc_bh = bh;
      ++acc_n;
      continue;
    }
    // ---- B: once every A item of the head is done, the codes
    if (acc_n > 0 && acc_bh <= bh) flush();  // never wait for a head while holding unmerged A items of it or of an earlier head
    if (tid == 0) {
      bool ok = *reinterpret_cast<volatile int*>(status) == 0;
      uint32_t i = 0;
      while (ok && ld_acquire(done + bh) < (unsigned int)g.nb) {
        if (++i > spin) { ok = false; atomicOr(status, 1); }
        __nanosleep(64);
      }
      *s_go = ok ? 1 : 0;
    }
    __syncthreads();
    if (!*s_go) continue;  // a wait gave up: the status word says so; the ring still drains
    const size_t blk_lin = (size_t)bh * g.nb + blk;
    const unsigned int* amax_bits = P.amax_bits + (size_t)bh * D;
    if (blk == 0 && tid < D) {
      const float a = __uint_as_float(__ldcg(amax_bits + tid));
      if (want_i8) P.s8[(size_t)bh * D + tid] = a > 0.f ? __fdiv_rn(a, 127.0f) : 0.f;
      if (want_f4) P.g4[(size_t)bh * D + tid] = __fdiv_rn(a, 2688.0f);
    }
    if (!active) continue;
    const float am0 = __uint_as_float(__ldcg(amax_bits + c0)), am1 = __uint_as_float(__ldcg(amax_bits + c0 + 1));
    if (want_i8) {
      // the codes of channels c0, c0+1 for this thread's 16 slots, as bf16
      // values (integers up to 127: exact), in the block's [slot][channel]
      // order — the layout of a bf16 V tile, so the INT8 phase's P·V runs on
      // the same tensor-core path as the 16-bit phase's
      const float inv0 = am0 > 0.f ? __fdiv_rn(127.0f, am0) : 0.f, inv1 = am1 > 0.f ? __fdiv_rn(127.0f, am1) : 0.f;
      __nv_bfloat16* dst = P.q8 + (blk_lin * 64 + 16 * j) * D + c0;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int k0 = max(-127, min(127, __float2int_rn(__fmul_rn(f0[e], inv0))));
        const int k1 = max(-127, min(127, __float2int_rn(__fmul_rn(f1[e], inv1))));
        *reinterpret_cast<__nv_bfloat162*>(dst + (size_t)e * D) =
            __floats2bfloat162_rn((float)k0, (float)k1);
      }
    }
    if (want_f4) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float* f = h ? f1 : f0;
        const int c = c0 + h;
        const float gch = __fdiv_rn(h ? am1 : am0, 2688.0f);
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
  flush();  // the last head's A items, if the items ran out after them
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
  // the preparation's status word is cleared by every call, V packed or not
  int* status = at<int>(ws, L, R_STATUS) + 1;
  if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, sizeof(int), st);
  if (e != cudaSuccess || !(want_i8 || want_f4)) return e;

  // the absmax words, then the work counter and one done counter per head (zero)
  unsigned int* amax = at<unsigned int>(ws, L, R_V_AMAX);
  unsigned int* work = amax + (size_t)g.BH * D;
  unsigned int* done = work + 1;
  e = cudaMemsetAsync(amax, 0, L.size[R_V_AMAX], st);
  if (e != cudaSuccess) return e;
  if (2LL * g.BH * g.nb > 0x7fffffffLL) return cudaErrorNotSupported;
  VPtrs V{static_cast<const __nv_bfloat16*>(v), amax, at<__nv_bfloat16>(ws, L, R_V_I8),
          at<float>(ws, L, R_V_S8), at<uint8_t>(ws, L, R_V_F4), at<uint8_t>(ws, L, R_V_SF4),
          at<float>(ws, L, R_V_G4)};
  CUtensorMap tv;
  if (!make_region_map(&tv, v, g, false)) return cudaErrorNotSupported;  // no tensor-map encoder in this driver
  using LY = PrepTmaLayout<D>;
  e = cudaFuncSetAttribute(v_prep_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::TOTAL);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, v_prep_kernel<D>, kThreads, LY::TOTAL);
  const int n_items = 2 * g.BH * g.nb;
  const int grid = std::max(1, std::min(n_items, sms * std::max(per_sm, 1)));
  v_prep_kernel<D><<<grid, kThreads, LY::TOTAL, st>>>(tv, g, V, want_i8, want_f4, n_items, work, done, status,
                                                      kPrepSpin);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prepare(const Geom& g, const Layout& L, const void* q, const void* k,
                           const void* v, void* ws, cudaStream_t st) {
  return g.d == 128 ? launch_prepare_d<128>(g, L, q, k, v, ws, st)
                    : launch_prepare_d<64>(g, L, q, k, v, ws, st);
}

}  // namespace da2
