// Stage 3 on the Blackwell tensor cores (tcgen05 + TMEM + TMA).
//
// DraftAttention2 abstract and reading note (Method overview bullet 4): one
// kernel runs a phase per precision for each query block, sharing data
// movement, softmax statistics and one output accumulator, and rescaling by the
// quantisation scales at phase boundaries.  DraftAttention (v1) abstract: the
// output is restored to the original token order.
//
// Tile shape.  A precision is assigned per (query block, key block) pair of 64
// tokens each, so a single query block gives an M = 64 MMA, which runs the
// tensor core at half rate.  Instead each CTA owns a pair of neighbouring query
// blocks (2p, 2p+1) — rows 0-63 and 64-127 of one M = 128 tile — and walks the
// merged, ordered key list of the pair, phase by phase.  A key block that only
// one of the two query blocks keeps in a phase is computed for all 128 rows
// and the other half's P rows are zero; on the video workloads 74-80 % of the
// computed rows are useful, against 50 % for M = 64.
//
// Units: every phase takes its key blocks two at a time (a, b).  Roles (10
// warps): warps 0-7 softmax — warp w owns TMEM lanes 32(w&3).. (tile rows),
// key block h = w>>2 of every unit (all 64 keys of it) and channels 64h..64h+63
// of the output; warp 8 issues TMA loads; warp 9 issues the MMAs from a
// non-blocking scheduler that starts S of a unit as soon as its buffers are
// free, ahead of the P·V of the unit before.
//   16-bit  S = Q·K^T (kind::f16 bf16, M128 N128, fp32 TMEM, 2 buffers);
//           P = exp2(s·log2e/√d − m_ref) rounded to bf16, m_ref an integer
//           exponent shared by the two warps of a row and raised lazily (O
//           rescaled in TMEM by a power of two only when the row max grows by
//           more than 2^8).  P replaces the warp's own scores in TMEM and
//           O += P·V reads it from there as the A operand (kind::f16, V read
//           MN-major from the TMA tile), so the softmax of a unit never waits
//           for the P·V of the one before unless O must be rescaled.
//   Low-bit phases accumulate P·V in TMEM at column 384 (INT8: s32 X8; 4-bit:
//   fp32 O4) against a power-of-two reference 2^r per row, shared by the two
//   warps of the row, starting from ceil of the row's running max over all
//   earlier units (the shared softmax statistics) and raised to ceil(unit
//   max) whenever a unit's max exceeds it; P is quantised relative to 2^r.  Before a raise (INT8 also
//   every 256 units, ahead of s32 overflow) and at the end of the phase the
//   accumulator is folded into O with the phase's channel scale (sv/255 or
//   g/2688) and cleared.
//   8-bit   S = Q8·[K8_a; K8_b]^T (kind::i8, s32); the row max is taken on
//           the integers, the exact fp32 scores (through the mantissa of
//           1.5·2^23) only after the max exchange; codes rint(255 p) as u8
//           replace the scores in TMEM; X8 += P8·V8 (kind::i8 u8×s8, A from
//           TMEM).
//   4-bit   S_h = Q4·K4_h^T (kind::mxf4nvf4, block16 e4m3 scales copied into
//           TMEM with tcgen05.cp from the scale atoms prep wrote); 2688 p
//           quantised to NVFP4 per 16 keys in registers, codes and scale atom
//           to shared memory; O4 += P4·V4 (block-scaled).
// Operands arrive by TMA: bf16 Q/K/V as 8×8-token region boxes straight from
// the [B,H,N,d] tensors (padding is the TMA zero fill), INT8 codes as 2-D
// boxes of the workspace.  The epilogue writes O through the same region box
// with a TMA store, whose clipping drops the padding rows — the restore.
// Every mbarrier wait is bounded; on expiry the CTA raises the workspace status
// word, skips the rest and releases its tensor memory.
#include <cuda.h>

#include <mutex>
#include <type_traits>

#include "da2_internal.cuh"
#include "sm100.cuh"

namespace da2 {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kSoftmaxWarps = 8;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr int kStages = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// INT8 MMAs accumulate onto the bit pattern of 1.5*2^23: an s32 result x
// (|x| < 2^22) then reads as the float 1.5*2^23 + x, exact, and one
// subtraction turns it into x.
constexpr uint32_t kI8Bias = 0x4B400000u;
constexpr float kI8BiasF = 12582912.0f;
// the 4-bit phase quantises 2688 p: 6 (largest e2m1) x 448 (largest e4m3)
constexpr float kP4Range = 2688.0f;

// shared-memory map (offsets from a 1024-aligned base)
constexpr uint32_t SM_Q16 = 0;         // [2 halves][128 rows][128 B], SW128
constexpr uint32_t SM_Q8 = 32768;      // [128 rows][128 B], SW128
constexpr uint32_t SM_K = 49152;       // K ring: kStages x 32 KB
constexpr uint32_t SM_V = SM_K + kStages * 32768;            // V ring: kStages x 32 KB
// 16-bit unit: K slot = K_a h0 | K_b h0 | K_a h1 | K_b h1 (8 KB each, so each
// channel half of [K_a; K_b] is one 128-row K-major operand); V slot = V_a | V_b
// (16 KB each).  INT8 unit: K slot = K8_a | K8_b (8 KB each: one 128-row
// operand), V slot = V8_a^T | V8_b^T (8 KB each).  4-bit unit: K slot =
// K4_a | K4_b ([64][64 B] SW64, 4 KB each) with their scale atoms (2 x 512 B
// per block) at +8192; V slot = V4_a^T | V4_b^T ([128][32 B] SW32, 4 KB each)
// with one scale atom per block at +8192.
constexpr uint32_t SL_SF = 8192;
// P area (4-bit units only; 16-bit and INT8 P stay in TMEM): P4_a | P4_b
// (4 KB each) at +0, their scale atoms at +16384.
constexpr uint32_t SM_P = SM_V + kStages * 32768;
constexpr uint32_t PO_PSF = 16384;
// channel scales that fold a low-bit accumulator into O (fp32 [128] each):
// INT8 sv/255 (P codes are 255 p) | NVFP4 g/2688 (P is quantised as 2688 p)
constexpr uint32_t SM_VS = SM_P + 32768;
constexpr uint32_t VS_SV255 = 0, VS_G2688 = 512;
constexpr uint32_t SM_RED = SM_VS + 1024;                    // row-statistics exchange, 4 KB
constexpr uint32_t SM_BAR = SM_RED + 4096;                   // mbarriers
constexpr uint32_t SM_MISC = SM_BAR + 512;
constexpr uint32_t SM_Q4 = (SM_MISC + 128 + 1023) & ~1023u;  // NVFP4 Q of the pair [128][64 B], SW64
constexpr uint32_t SM_TOTAL = SM_Q4 + 8192;
constexpr uint32_t kSmemBytes = SM_TOTAL + 1024;  // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// TMEM columns: O 0-127 (every phase); S 2 x 128 at 128 (16-bit and INT8
// units; a 4-bit unit uses one, S_a 128 and S_b 192); the low-bit phase
// accumulator at 384 (INT8 s32 X8, then 4-bit fp32 O4); 4-bit scale factors
// from 256 — Q 256, K_a 264, K_b 272, V_a 280, V_b 284, P_a 288, P_b 292, all
// 4-aligned as block-scaled MMAs require.
constexpr uint32_t TM_O = 0, TM_S = 128, TM_ACC = 384;
constexpr uint32_t TM_SFQ = 256, TM_SFK = 264, TM_SFV = 280, TM_SFP = 288;

// mbarrier slots (8 bytes each)
enum {
  B_Q16 = 0, B_Q8, B_Q4, B_SFQ, B_K_FULL, B_K_EMPTY = B_K_FULL + kStages, B_V_FULL = B_K_EMPTY + kStages,
  B_V_EMPTY = B_V_FULL + kStages, B_S_FULL = B_V_EMPTY + kStages,
  B_S_FREE = B_S_FULL + 2, B_P_FULL = B_S_FREE + 2, B_P_FREE = B_P_FULL + 2, B_DONE = B_P_FREE + 2,
  B_PAIR = B_DONE + 1,   // [4 quarters][2 parities]: the two warps of a row quarter
  B_EPI = B_PAIR + 8,    // [4 quarters]: final exchange
  B_COUNT = B_EPI + 4
};
static_assert(B_COUNT * 8 <= 512, "barrier area");

struct TcArgs {
  const uint32_t* plist;  // [BH][npairs][2*nb]
  const int* pcnt;        // [BH][npairs][4]
  const float* q_s8;
  const float* k_s8;
  const float* v_s8;
  const float* v_g4;
  const uint8_t* q_sf4;
  const uint8_t* k_sf4;
  const uint8_t* v_sf4;
  int* status;
  int npairs;
};

__device__ __forceinline__ void raise_timeout(int* status) { atomicOr(status, 1); }

// packed fp32x2 arithmetic (one FMA-pipe instruction for two lanes' values)
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// bytes 0 of four words -> one word (x0 in the low byte)
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3) {
  uint32_t lo, hi, r;
  asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(lo) : "r"(x0), "r"(x1));
  asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(hi) : "r"(x2), "r"(x3));
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(r) : "r"(lo), "r"(hi));
  return r;
}

// Items: kb | inA << 16 | inB << 17 | kind << 18 (kind 0 = 16-bit, 1 = 8-bit)
//        | full << 20 (the key block has no padding slot).
__device__ __forceinline__ int item_kb(uint32_t e) { return (int)(e & 0xffffu); }

__device__ __forceinline__ bool item_full(uint32_t e) { return (e >> 20) & 1u; }

__device__ __forceinline__ unsigned long long key_mask(const Geom& g, int kb) {
  const int rx = kb % g.nrx, ry = (kb / g.nrx) % g.nry;
  const int vy = min(g.rh, g.Hh - ry * g.rh), vx = min(g.rw, g.Ww - rx * g.rw);
  if (vy == g.rh && vx == g.rw) return ~0ull;
  const unsigned long long rowbits = (vx >= 64) ? ~0ull : ((1ull << vx) - 1ull);
  unsigned long long m = 0;
  for (int i = 0; i < vy; ++i) m |= rowbits << (g.rw * i);
  return m;
}

// kDense: every key block in the 16-bit phase, no item lists read (a separate
// instantiation, so that the sparse kernel carries none of it)
template <bool kDense>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const __grid_constant__ CUtensorMap tmQ8, const __grid_constant__ CUtensorMap tmK8,
               const __grid_constant__ CUtensorMap tmV8, const __grid_constant__ CUtensorMap tmQ4,
               const __grid_constant__ CUtensorMap tmK4, const __grid_constant__ CUtensorMap tmV4, Geom g,
               TcArgs A) {
  // a CTA that timed out raised the status word: later CTAs skip their work
  if (*reinterpret_cast<volatile const int*>(A.status) != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s0 = (uint32_t)__cvta_generic_to_shared(smem);
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qa = 2 * pair, qb = (2 * pair + 1 < g.nb) ? 2 * pair + 1 : -1;
  const size_t prow = (size_t)bh * A.npairs + pair;
  const int4 pc = kDense ? make_int4(g.nb, 0, 0, 0) : *reinterpret_cast<const int4*>(A.pcnt + prow * 4);
  const int n16 = pc.x, n8 = pc.y, n4 = pc.z;
  const uint32_t* items = kDense ? nullptr : A.plist + prow * (size_t)(2 * g.nb);
  // entry i of the pair's list; in dense mode key block i, kept by both query
  // blocks, flagged full unless it holds the ragged tail
  auto item_at = [&](int i) -> uint32_t {
    if (!kDense) return items[i];
    return (uint32_t)i | (1u << 16) | ((2 * pair + 1 < g.nb ? 1u : 0u) << 17) |
           ((uint32_t)((i + 1) * 64 <= g.N) << 20);
  };
  auto bar = [&](int i) { return s0 + SM_BAR + 8u * (uint32_t)i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + SM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM_MISC + 8);
  // 1 / (1 + m/8) for m = 0..7, then 1 / m (0 for m = 0): reciprocals of e4m3 scales
  float* rcp_tab = reinterpret_cast<float*>(smem + SM_MISC + 64);
  if (threadIdx.x < 16)
    rcp_tab[threadIdx.x] = threadIdx.x < 8 ? 8.0f / (float)(8 + threadIdx.x)
                                           : (threadIdx.x > 8 ? 1.0f / (float)(threadIdx.x - 8) : 0.f);

  // units: each phase takes its items (key blocks) two at a time, in list order
  const int nu16 = (n16 + 1) / 2;
  const int nu8 = nu16 + (n8 + 1) / 2;  // INT8 units end here, 4-bit units follow
  const int nu = nu8 + (n4 + 1) / 2;
  auto unit_items = [&](int u, int& i0, int& cnt) {
    if (u < nu16) { i0 = 2 * u; cnt = min(2, n16 - i0); }
    else if (u < nu8) { i0 = n16 + 2 * (u - nu16); cnt = min(2, n16 + n8 - i0); }
    else { i0 = n16 + n8 + 2 * (u - nu8); cnt = min(2, n16 + n8 + n4 - i0); }
  };


  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q16), 1);
    mbar_init(bar(B_Q8), 1);
    mbar_init(bar(B_Q4), 1);
    mbar_init(bar(B_SFQ), 4);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_K_FULL + s), 1); mbar_init(bar(B_K_EMPTY + s), 1);
      mbar_init(bar(B_V_FULL + s), 1); mbar_init(bar(B_V_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_S_FULL + b), 1);
      mbar_init(bar(B_S_FREE + b), kSoftmaxWarps);
    }
    for (int b = 0; b < 2; ++b) {  // per unit parity: P of unit u, P·V of unit u
      mbar_init(bar(B_P_FULL + b), kSoftmaxWarps);
      mbar_init(bar(B_P_FREE + b), 1);
    }
    mbar_init(bar(B_DONE), 1);
    for (int i = 0; i < 8; ++i) mbar_init(bar(B_PAIR + i), 2);
    for (int i = 0; i < 4; ++i) mbar_init(bar(B_EPI + i), 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(s0 + SM_MISC, 512);
  if (threadIdx.x < kD && !kDense) {
    const float sv = A.v_s8[(size_t)bh * kD + threadIdx.x], gv = A.v_g4[(size_t)bh * kD + threadIdx.x];
    float* vsc = reinterpret_cast<float*>(smem + SM_VS);
    vsc[VS_SV255 / 4 + threadIdx.x] = sv / 255.0f;
    vsc[VS_G2688 / 4 + threadIdx.x] = gv / kP4Range;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];
  if (warp < kSoftmaxWarps) {
    // the low-bit accumulator starts at zero
    const uint32_t own = tbase + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(warp >> 2) * 64;
    bool any = false;
    if (n8 > 0 || n4 > 0) {  // the low-bit accumulator starts at zero
      tmem_fill32(own + TM_ACC, 0u);
      tmem_fill32(own + TM_ACC + 32, 0u);
      any = true;
    }
    if (any) tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int t_of = g.nry * g.nrx;  // blocks per frame
  auto box = [&](int blk, int& cx, int& cy, int& cf) {
    const int t = blk / t_of, rem = blk - t * t_of;
    const int ry = rem / g.nrx, rx = rem - ry * g.nrx;
    cx = rx * g.rw; cy = ry * g.rh; cf = bh * g.T + t;
  };

  if (warp == kProducerWarp) {
    // ---------------------------------------------------------------- TMA producer
    if (elect_one()) {
      prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmV);
      int cx, cy, cf;
      if (n16 > 0) {
        mbar_expect_tx(bar(B_Q16), qb >= 0 ? 32768u : 16384u);
        box(qa, cx, cy, cf);
        tma_load_4d(s0 + SM_Q16, &tmQ, bar(B_Q16), 0, cx, cy, cf);
        tma_load_4d(s0 + SM_Q16 + 16384, &tmQ, bar(B_Q16), 64, cx, cy, cf);
        if (qb >= 0) {
          box(qb, cx, cy, cf);
          tma_load_4d(s0 + SM_Q16 + 8192, &tmQ, bar(B_Q16), 0, cx, cy, cf);
          tma_load_4d(s0 + SM_Q16 + 16384 + 8192, &tmQ, bar(B_Q16), 64, cx, cy, cf);
        }
      }
      if (n8 > 0) {
        mbar_expect_tx(bar(B_Q8), qb >= 0 ? 16384u : 8192u);
        tma_load_2d(s0 + SM_Q8, &tmQ8, bar(B_Q8), 0, (bh * g.nb + qa) * 64);
        if (qb >= 0) tma_load_2d(s0 + SM_Q8 + 8192, &tmQ8, bar(B_Q8), 0, (bh * g.nb + qb) * 64);
      }
      if (n4 > 0) {
        mbar_expect_tx(bar(B_Q4), qb >= 0 ? 8192u : 4096u);
        tma_load_2d(s0 + SM_Q4, &tmQ4, bar(B_Q4), 0, (bh * g.nb + qa) * 64);
        if (qb >= 0) tma_load_2d(s0 + SM_Q4 + 4096, &tmQ4, bar(B_Q4), 0, (bh * g.nb + qb) * 64);
      }
      // K of a unit is needed first (scores) and released first; V waits for
      // the P·V two units back.  Issue whichever ring has room, K first.
      int kn = 0, vn = 0;
      uint32_t idle = 0;
      while (kn < nu || vn < nu) {
        bool progressed = false;
        if (kn < nu && (kn < kStages || mbar_test(bar(B_K_EMPTY + kn % kStages), ((kn / kStages) - 1) & 1))) {
          int i0, cnt;
          unit_items(kn, i0, cnt);
          const uint32_t dst = s0 + SM_K + (kn % kStages) * 32768;
          const uint32_t fb = bar(B_K_FULL + kn % kStages);
          if (kn < nu16) {
            mbar_expect_tx(fb, 16384u * (uint32_t)cnt);
            for (int t = 0; t < cnt; ++t) {
              box(item_kb(item_at(i0 + t)), cx, cy, cf);
              tma_load_4d(dst + t * 8192, &tmK, fb, 0, cx, cy, cf);
              tma_load_4d(dst + 16384 + t * 8192, &tmK, fb, 64, cx, cy, cf);
            }
          } else if (kn < nu8) {
            mbar_expect_tx(fb, 8192u * (uint32_t)cnt);
            for (int t = 0; t < cnt; ++t)
              tma_load_2d(dst + t * 8192, &tmK8, fb, 0, (bh * g.nb + item_kb(item_at(i0 + t))) * 64);
          } else {
            mbar_expect_tx(fb, (4096u + 2 * kSfAtomBytes) * (uint32_t)cnt);
            for (int t = 0; t < cnt; ++t) {
              const size_t kl = (size_t)bh * g.nb + item_kb(item_at(i0 + t));
              tma_load_2d(dst + t * 4096, &tmK4, fb, 0, (int)(kl * 64));
              bulk_load(dst + SL_SF + t * 2 * kSfAtomBytes, A.k_sf4 + kl * 2 * kSfAtomBytes, 2 * kSfAtomBytes, fb);
            }
          }
          ++kn;
          progressed = true;
        }
        if (vn < kn && (vn < kStages || mbar_test(bar(B_V_EMPTY + vn % kStages), ((vn / kStages) - 1) & 1))) {
          int i0, cnt;
          unit_items(vn, i0, cnt);
          const uint32_t dst = s0 + SM_V + (vn % kStages) * 32768;
          const uint32_t fb = bar(B_V_FULL + vn % kStages);
          if (vn < nu16) {
            mbar_expect_tx(fb, 16384u * (uint32_t)cnt);
            for (int t = 0; t < cnt; ++t) {
              box(item_kb(item_at(i0 + t)), cx, cy, cf);
              tma_load_4d(dst + t * 16384, &tmV, fb, 0, cx, cy, cf);
              tma_load_4d(dst + t * 16384 + 8192, &tmV, fb, 64, cx, cy, cf);
            }
          } else if (vn < nu8) {
            mbar_expect_tx(fb, 8192u * (uint32_t)cnt);
            for (int t = 0; t < cnt; ++t)
              tma_load_2d(dst + t * 8192, &tmV8, fb, 0, (bh * g.nb + item_kb(item_at(i0 + t))) * kD);
          } else {
            mbar_expect_tx(fb, (4096u + kSfAtomBytes) * (uint32_t)cnt);
            for (int t = 0; t < cnt; ++t) {
              const size_t kl = (size_t)bh * g.nb + item_kb(item_at(i0 + t));
              tma_load_2d(dst + t * 4096, &tmV4, fb, 0, (int)(kl * kD));
              bulk_load(dst + SL_SF + t * kSfAtomBytes, A.v_sf4 + kl * kSfAtomBytes, kSfAtomBytes, fb);
            }
          }
          ++vn;
          progressed = true;
        }
        if (progressed) {
          idle = 0;
        } else if (++idle > (1u << 24) || *abort_flag) {
          raise_timeout(A.status); *abort_flag = 1;
          break;
        } else {
          __nanosleep(64);  // leave the issue slots of this sub-partition to the softmax warps
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA scheduler
    if (elect_one()) {
      const uint32_t id16n128 = idesc(kDF32, kFmtBF16, kFmtBF16, false, false, 128, 128);
      const uint32_t id16n64 = idesc(kDF32, kFmtBF16, kFmtBF16, false, false, 128, 64);
      const uint32_t idpv = idesc(kDF32, kFmtBF16, kFmtBF16, false, true, 128, 128);
      const uint32_t id8n64 = idesc(kDS32, kFmtS8, kFmtS8, false, false, 128, 64);
      const uint32_t id8n128 = idesc(kDS32, kFmtS8, kFmtS8, false, false, 128, 128);
      const uint32_t idx8 = idesc(kDS32, kFmtU8, kFmtS8, false, false, 128, 128);
      const uint32_t id4s = idesc_f4(128, 64), id4pv = idesc_f4(128, 128);
      bool f4_ready = false;  // Q4 loaded and its scales in TMEM
      bool ok = true;
      if (n16 > 0) ok = ok && mbar_wait(bar(B_Q16), 0);
      if (n8 > 0) ok = ok && mbar_wait(bar(B_Q8), 0);
      int sn = 0, pn = 0;  // next unit for S, next unit for P·V
      uint32_t idle = 0;
      while (ok && pn < nu) {
        bool progressed = false;
        if (sn < nu) {
          const int s = sn % kStages, b = sn & 1;
          const bool single = sn >= nu8;
          if (single && !f4_ready) {
            // first 4-bit unit: Q4 must be in shared memory and its scales in TMEM
            f4_ready = mbar_test(bar(B_Q4), 0) && mbar_test(bar(B_SFQ), 0);
          }
          // 16-bit and INT8 units alternate two S buffers and leave their P
          // there until their P·V completes; 4-bit units share one (the
          // second holds scale factors), so they wait for the unit before —
          // for the first of them that implies both buffers were read
          auto pv_done = [&](int j) {
            return j < 0 || j >= nu8 || mbar_test(bar(B_P_FREE + (j & 1)), (j >> 1) & 1);
          };
          const bool s_free = single ? (sn < 1 || mbar_test(bar(B_S_FREE + ((sn - 1) & 1)), ((sn - 1) >> 1) & 1)) &&
                                           pv_done(sn - 1) && pv_done(sn - 2)
                                     : (sn < 2 || mbar_test(bar(B_S_FREE + b), ((sn >> 1) - 1) & 1)) && pv_done(sn - 2);
          if ((sn < nu8 || f4_ready) && s_free && mbar_test(bar(B_K_FULL + s), (sn / kStages) & 1)) {
            tc_fence_after();
            const uint32_t st = s0 + SM_K + s * 32768;
            const uint32_t sd = tbase + TM_S + (single ? 0u : b * 128u);
            int i0, cnt;
            unit_items(sn, i0, cnt);
            if (sn < nu16) {
              const uint32_t id = cnt == 2 ? id16n128 : id16n64;
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int h = k >> 2, kk = k & 3;
                mma_f16(sd, smem_desc(s0 + SM_Q16 + h * 16384 + kk * 32, 16, 1024, SW_128),
                        smem_desc(st + h * 16384 + kk * 32, 16, 1024, SW_128), id, k > 0 ? 1u : 0u);
              }
            } else if (sn < nu8) {
              const uint32_t id = cnt == 2 ? id8n128 : id8n64;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_i8(sd, smem_desc(s0 + SM_Q8 + kk * 32, 16, 1024, SW_128),
                       smem_desc(st + kk * 32, 16, 1024, SW_128), id,
                       kk > 0 ? 1u : 0u);
            } else {
              for (int t = 0; t < cnt; ++t) {
                const uint32_t sfk = tbase + TM_SFK + 8 * t;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                  tc_cp_atom(sfk + 4 * c, st + SL_SF + (2 * t + c) * kSfAtomBytes);
                  mma_f4(sd + 64 * t, smem_desc(s0 + SM_Q4 + 32 * c, 16, 512, SW_64),
                         smem_desc(st + t * 4096 + 32 * c, 16, 512, SW_64), id4s, c > 0 ? 1u : 0u,
                         tbase + TM_SFQ + 4 * c, sfk + 4 * c);
                }
              }
            }
            mma_commit(bar(B_S_FULL + b));
            mma_commit(bar(B_K_EMPTY + s));
            ++sn;
            progressed = true;
          }
        }
        if (pn < sn) {
          const int s = pn % kStages;
          const bool low = pn >= nu16;  // INT8 or 4-bit: P·V accumulates at TM_ACC
          // (the softmax warps settle the accumulator before they release P)
          if (mbar_test(bar(B_V_FULL + s), (pn / kStages) & 1) &&
              mbar_test(bar(B_P_FULL + (pn & 1)), (pn >> 1) & 1)) {
            tc_fence_after();
            const uint32_t st = s0 + SM_V + s * 32768;
            const uint32_t pbuf = s0 + SM_P;
            if (!low) {
              int i0, cnt;
              unit_items(pn, i0, cnt);
              // P of block t sits in TMEM, in block t's own score columns
              const uint32_t pt = tbase + TM_S + (pn & 1) * 128;
              for (int t = 0; t < cnt; ++t) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_f16_ta(tbase + TM_O, pt + 64 * t + 8 * kk,
                             smem_desc(st + t * 16384 + kk * 2048, 8192, 1024, SW_128), idpv, 1u);
              }
            } else if (pn < nu8) {
              int i0, cnt;
              unit_items(pn, i0, cnt);
              for (int t = 0; t < cnt; ++t) {
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                  mma_i8_ta(tbase + TM_ACC, tbase + TM_S + (pn & 1) * 128 + 64 * t + 8 * kk,
                            smem_desc(st + t * 8192 + kk * 32, 16, 512, SW_64), idx8, 1u);
              }
            } else {
              int i0, cnt;
              unit_items(pn, i0, cnt);
              for (int t = 0; t < cnt; ++t) {
                const uint32_t sfv = tbase + TM_SFV + 4 * t, sfp = tbase + TM_SFP + 4 * t;
                tc_cp_atom(sfv, st + SL_SF + t * kSfAtomBytes);
                tc_cp_atom(sfp, pbuf + PO_PSF + t * kSfAtomBytes);
                mma_f4(tbase + TM_ACC, smem_desc(pbuf + t * 4096, 16, 256, SW_32),
                       smem_desc(st + t * 4096, 16, 256, SW_32), id4pv, 1u, sfp, sfv);
              }
            }
            mma_commit(bar(B_P_FREE + (pn & 1)));
            mma_commit(bar(B_V_EMPTY + s));
            ++pn;
            progressed = true;
          }
        }
        if (progressed) {
          idle = 0;
        } else if (++idle > (1u << 24) || *abort_flag) {
          ok = false;
        } else {
          __nanosleep(32);  // leave the issue slots of this sub-partition to the softmax warps
        }
      }
      mma_commit(bar(B_DONE));
      if (!ok) { raise_timeout(A.status); *abort_flag = 1; }
    }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-7
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;  // TMEM lane and tile row
    const bool in_b = row >= 64;
    const int qrow_blk = in_b ? qb : qa;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = kLog2e * rsqrtf((float)kD);
    const float sq = (n8 > 0 && qrow_blk >= 0) ? A.q_s8[(size_t)bh * g.nb + qrow_blk] : 0.f;
    float* red = reinterpret_cast<float*>(smem + SM_RED);  // [2][2][128]
    const unsigned FULL = 0xffffffffu;
    // the two warps of a row quarter exchange row statistics through shared
    // memory, ordered by an mbarrier (bounded wait, unlike a named barrier)
    auto pair_sync = [&](int idx, uint32_t parity) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(idx));
      return __all_sync(FULL, mbar_wait(bar(idx), parity));
    };
    // the P·V of unit v (and every MMA before it) has completed
    auto pfree_wait = [&](int v) -> bool {
      return v < 0 || mbar_wait(bar(B_P_FREE + (v & 1)), (uint32_t)(v >> 1) & 1u);
    };
    float m16 = -INFINITY, l16 = 0.f;  // 16-bit phase: O in TMEM, integer reference
    float x_run = -INFINITY;            // running row max (log2 units) over every unit so far
    bool ok = true;
    {  // O starts at zero (this warp's 64 columns)
      uint32_t z[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = 0u;
      tmem_st32(tbase + lane_off + TM_O + half * 64, z);
      tmem_st32(tbase + lane_off + TM_O + half * 64 + 32, z);
      tmem_wait_st();
    }
    // item entries (and INT8 key scales) are loaded one unit ahead, so no unit
    // starts by waiting on global memory
    auto item_for = [&](int v) -> uint32_t {
      if (v >= nu) return 0u;
      int i0v, cntv;
      unit_items(v, i0v, cntv);
      return half < cntv ? item_at(i0v + half) : 0u;
    };
    auto sk_for = [&](int v, uint32_t ev) -> float {
      return (v >= nu16 && v < nu8) ? A.k_s8[(size_t)bh * g.nb + item_kb(ev)] : 0.f;
    };
    uint32_t e_next = item_for(0);
    float sk_next = sk_for(0, e_next);
    for (int u = 0; ok && u < nu16; ++u) {
      if ((u & 7) == 0 && __any_sync(FULL, *abort_flag != 0)) { ok = false; break; }
      const int b = u & 1;
      int i0, cnt;
      unit_items(u, i0, cnt);
      float* xch = red + (u & 1) * 256;  // [2 halves][128 rows] for this unit
      const uint32_t sbase = tbase + lane_off + TM_S + b * 128;
      if (!__all_sync(FULL, mbar_wait(bar(B_S_FULL + b), (u >> 1) & 1))) { ok = false; break; }
      tc_fence_after();
        // ---- 16-bit unit: this warp owns key block `half` of the unit
        const bool present = half < cnt;
        const uint32_t e = e_next;
        e_next = item_for(u + 1);
        const bool member = present && (((e >> (in_b ? 17 : 16)) & 1u) != 0);
        uint32_t sr[64];
        if (present) {
          tmem_ld32(sbase + half * 64, sr);
          tmem_ld32(sbase + half * 64 + 32, sr + 32);
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_FREE + b));
        float mx = -INFINITY;
        if (member) {
          if (!item_full(e)) {
            const unsigned long long vm = key_mask(g, item_kb(e));
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (!((vm >> i) & 1ull)) sr[i] = __float_as_uint(-INFINITY);
          }
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int i = 0; i < 64; i += 8)
#pragma unroll
            for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], __uint_as_float(sr[i + 2 * q]), __uint_as_float(sr[i + 2 * q + 1]));
          mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
        }
        xch[half * 128 + row] = mx;
        if (!pair_sync(B_PAIR + quarter * 2 + (u & 1), (u >> 1) & 1)) { ok = false; break; }
        sk_next = sk_for(u + 1, e_next);  // the entry has arrived by now; the scale has a unit's time
        mx = fmaxf(mx, xch[(1 - half) * 128 + row]) * sl2;  // unit row max, log2 units
        const bool row_live = mx != -INFINITY;  // the row is a member of some block of the unit
        x_run = fmaxf(x_run, mx);
        const bool need = row_live && (mx > m16 + kRescaleThreshold || m16 == -INFINITY);
        const bool need_o = need && m16 != -INFINITY;
        const float a = need_o ? ldexpf(1.0f, (int)(m16 - ceilf(mx))) : 1.0f;
        if (need) m16 = ceilf(mx);
        // P of this warp's block, ahead of the wait for the previous P·V
        uint32_t pw[32];
        if (member) {
          const uint64_t sl2x2 = f2pack(sl2, sl2), negm = f2pack(-m16, -m16);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float x0, x1;
            f2unpack(f2fma(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), sl2x2, negm), x0, x1);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            acc[i & 3] = f2add(acc[i & 3], f2pack(p0, p1));
            __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
            pw[i] = *reinterpret_cast<uint32_t*>(&hb);
          }
          float s0, s1, s2, s3, s4, s5, s6, s7;
          f2unpack(f2add(acc[0], acc[1]), s0, s1);
          f2unpack(f2add(acc[2], acc[3]), s2, s3);
          (void)s4; (void)s5; (void)s6; (void)s7;
          l16 = l16 * a + ((s0 + s1) + (s2 + s3));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) pw[i] = 0u;
          l16 *= a;
        }
        // O can be rescaled once the P·V of unit u-1 completed; only then wait
        if (__any_sync(FULL, need_o)) {
          if (!__all_sync(FULL, pfree_wait(u - 1))) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 64; c += 32) {
            uint32_t orr[32];
            tmem_ld32(tbase + lane_off + TM_O + half * 64 + c, orr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * a);
            tmem_st32(tbase + lane_off + TM_O + half * 64 + c, orr);
          }
          tmem_wait_st();
        }
        // P (bf16 pairs, key 2i in the low half of column i) replaces this
        // warp's own scores in TMEM, where the P·V MMA reads it
        if (present) {
          tmem_st32(sbase + half * 64, pw);
          tmem_wait_st();
        }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P_FULL + (u & 1)));
    }
    // ================================================================ low-bit phases
    // Each low-bit phase accumulates P·V in TMEM (INT8: s32 X8; 4-bit: fp32
    // O4, both at column 384) against its own power-of-two reference r per
    // row, shared by the two warps of the row; P is quantised relative to 2^r.
    // When a unit's row maximum exceeds r, the accumulator is first folded
    // into O with the phase's channel scale (sv/255 or g/2688) and cleared;
    // so is it at the end of the phase.  l_lo is this warp's partial sum of p
    // against the same reference.
    const float* chs8 = reinterpret_cast<const float*>(smem + SM_VS + VS_SV255);
    const float* chs4 = reinterpret_cast<const float*>(smem + SM_VS + VS_G2688);
    // the phases share the softmax statistics: a low-bit phase starts from the
    // ceiling of the running maximum of everything before it
    float r_lo = ceilf(x_run), l_lo = 0.f;
    // fold the phase accumulator (this warp's 64 channels) into O for the
    // lanes in `sel`; O's reference becomes max(m16, r_lo) for them
    auto fold = [&](bool sel, bool i8) {
      if (!__any_sync(FULL, sel)) return;
      float a16 = 1.f, ax = 0.f;
      if (sel && r_lo != -INFINITY) {
        const float R = fmaxf(m16, r_lo);
        a16 = m16 == -INFINITY ? 0.f : ldexpf(1.0f, (int)(m16 - R));
        ax = ldexpf(1.0f, (int)(r_lo - R));
        l16 = l16 * a16 + l_lo * ax;
        m16 = R;
      }
      if (sel) l_lo = 0.f;
      const float* chs = (i8 ? chs8 : chs4) + half * 64;
#pragma unroll 1
      for (int c = 0; c < 64; c += 16) {
        uint32_t orr[16], xr[16];
        tmem_ld16(tbase + lane_off + TM_O + half * 64 + c, orr);
        tmem_ld16(tbase + lane_off + TM_ACC + half * 64 + c, xr);
        tmem_wait_ld();
        if (sel) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float x = i8 ? __int2float_rn((int)xr[i]) : __uint_as_float(xr[i]);
            orr[i] = __float_as_uint(fmaf(x, ax * chs[c + i], __uint_as_float(orr[i]) * a16));
            xr[i] = 0u;  // s32 0 and fp32 +0 alike
          }
        }
        tmem_st16(tbase + lane_off + TM_O + half * 64 + c, orr);
        tmem_st16(tbase + lane_off + TM_ACC + half * 64 + c, xr);
      }
      tmem_wait_st();
    };
    // one low-bit unit, instantiated once per format so that each phase's
    // loop holds only its own code
    auto lowbit_unit = [&](const int u, auto fmt) -> bool {
      constexpr bool i8 = decltype(fmt)::value;
      if ((u & 7) == 0 && __any_sync(FULL, *abort_flag != 0)) return false;
      if (!i8 && u == nu8 && nu8 > nu16) {
        // INT8 -> 4-bit boundary: the INT8 accumulator joins O once its last
        // P·V completed; the columns then start the 4-bit accumulator at zero
        if (!__all_sync(FULL, pfree_wait(u - 1))) return false;
        tc_fence_after();
        fold(true, true);  // the reference carries on into the 4-bit phase
      }
      int i0, cnt;
      unit_items(u, i0, cnt);
      // ---- this warp's block of the unit: key block `half`, all 64 keys
      const bool present = half < cnt;
      const uint32_t e = e_next;
      const float sk = sk_next;
      e_next = item_for(u + 1);
      const int kb = item_kb(e);
      const bool member = present && (((e >> (in_b ? 17 : 16)) & 1u) != 0);
      if (!i8 && u == nu8 && half == 0) {
        // first 4-bit unit: Q's scale factors into TMEM (each lane quarter
        // holds all 128 rows).  The columns were the second S buffer, whose
        // scores this warp has read, and no S MMA writes there any more.
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t w[4];
          const uint8_t* sa = A.q_sf4 + ((size_t)bh * g.nb + qa) * 2 * kSfAtomBytes + c * kSfAtomBytes + lane * 16;
          w[0] = *reinterpret_cast<const uint32_t*>(sa);
          w[1] = *reinterpret_cast<const uint32_t*>(sa + 4);
          if (qb >= 0) {
            const uint8_t* sb = A.q_sf4 + ((size_t)bh * g.nb + qb) * 2 * kSfAtomBytes + c * kSfAtomBytes + lane * 16;
            w[2] = *reinterpret_cast<const uint32_t*>(sb);
            w[3] = *reinterpret_cast<const uint32_t*>(sb + 4);
          } else {
            w[2] = w[3] = 0u;
          }
          tmem_st4(tbase + lane_off + TM_SFQ + 4 * c, w);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_SFQ));
      }
      float* xch = red + (u & 1) * 256;  // [2 halves][128 rows] for this unit
      if (!__all_sync(FULL, mbar_wait(bar(B_S_FULL + (u & 1)), (u >> 1) & 1))) return false;
      tc_fence_after();
      // this warp's scores: 64 columns of the unit's S buffer
      const uint32_t scol = tbase + lane_off + TM_S + (i8 ? (uint32_t)(u & 1) * 128u : 0u) + half * 64;
      const unsigned long long vm = item_full(e) ? ~0ull : key_mask(g, kb);
      const bool full = vm == ~0ull;
      uint32_t sr[64];
      float mx = -INFINITY;
      const float sc = i8 ? sq * sk * sl2 : sl2;  // score scale, log2 units (INT8: >= 0)
      // member is uniform across the warp (its rows belong to one query block)
      if (member) {
        tmem_ld32(scol, sr);
        tmem_ld32(scol + 32, sr + 32);
        tmem_wait_ld();
        if (i8) {
          // the row max on the integer scores (padding keys at INT_MIN); their
          // conversion to fp32 waits until after the max exchange
          if (!full) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (!((vm >> i) & 1ull)) sr[i] = 0x80000000u;
          }
          int m4[4] = {INT_MIN, INT_MIN, INT_MIN, INT_MIN};
#pragma unroll
          for (int i = 0; i < 64; i += 8)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              m4[q] = max(m4[q], max((int)sr[i + 2 * q], (int)sr[i + 2 * q + 1]));
          mx = (float)max(max(m4[0], m4[1]), max(m4[2], m4[3])) * sc;  // a member row has a real key
        } else {
          if (!full) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (!((vm >> i) & 1ull)) sr[i] = __float_as_uint(-INFINITY);
          }
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int i = 0; i < 64; i += 8)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              m4[q] = fmax3(m4[q], __uint_as_float(sr[i + 2 * q]), __uint_as_float(sr[i + 2 * q + 1]));
          mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * sc;
        }
      }
      if (!i8) {  // 4-bit units share one S buffer: release it at once
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_FREE + (u & 1)));
      }
      xch[half * 128 + row] = mx;
      if (!pair_sync(B_PAIR + quarter * 2 + (u & 1), (u >> 1) & 1)) return false;
      sk_next = sk_for(u + 1, e_next);  // the entry has arrived by now; the scale has a unit's time
      mx = fmaxf(mx, xch[(1 - half) * 128 + row]);  // the unit's row maximum
      // the reference rises to ceil(max) whenever the max exceeds it
      const bool raise = mx != -INFINITY && (r_lo == -INFINITY || mx > r_lo);
      const float r_use = raise ? ceilf(mx) : r_lo;
      float lp = 0.f;  // this warp's sum of the unquantised p of the unit
      uint32_t pw[16];
      uint32_t sfw = 0u;  // 4-bit: the row's four e4m3 P scales
#pragma unroll
      for (int i = 0; i < 16; ++i) pw[i] = 0u;
      if (member) {
        const uint64_t scx2 = f2pack(sc, sc), negr = f2pack(-r_use, -r_use);
        uint64_t ls[4] = {0ull, 0ull, 0ull, 0ull};
        // p = exp2(s*sc - r) in place of the scores (INT8: the exact s32 ->
        // fp32 conversion first, through the mantissa of 1.5*2^23, |S| < 2^22)
        const uint64_t kx2 = f2pack(-kI8BiasF, -kI8BiasF);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          uint64_t sp = f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
          if (i8) sp = f2add(f2pack(__uint_as_float(sr[2 * i] + kI8Bias), __uint_as_float(sr[2 * i + 1] + kI8Bias)), kx2);
          float x0, x1;
          f2unpack(f2fma(sp, scx2, negr), x0, x1);
          float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          if (!full) {  // padding keys contribute nothing, whatever the block scale (sc may be 0)
            if (!((vm >> (2 * i)) & 1ull)) p0 = 0.f;
            if (!((vm >> (2 * i + 1)) & 1ull)) p1 = 0.f;
          }
          ls[i & 3] = f2add(ls[i & 3], f2pack(p0, p1));
          sr[2 * i] = __float_as_uint(p0);
          sr[2 * i + 1] = __float_as_uint(p1);
        }
        float s0, s1, s2, s3;
        f2unpack(f2add(ls[0], ls[1]), s0, s1);
        f2unpack(f2add(ls[2], ls[3]), s2, s3);
        lp = (s0 + s1) + (s2 + s3);
        if (i8) {
          const uint64_t c255 = f2pack(255.0f, 255.0f), kmag = f2pack(12582912.0f, 12582912.0f);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            uint32_t c[4];
#pragma unroll
            for (int q = 0; q < 4; q += 2) {
              float r0, r1;  // 255 p + 1.5*2^23: round-to-nearest-even code in the low byte
              f2unpack(f2fma(f2pack(__uint_as_float(sr[4 * i + q]), __uint_as_float(sr[4 * i + q + 1])), c255, kmag),
                       r0, r1);
              c[q] = __float_as_uint(r0);
              c[q + 1] = __float_as_uint(r1);
            }
            pw[i] = pack_low_bytes(c[0], c[1], c[2], c[3]);
          }
        } else {
          // NVFP4 of 2688 p over 16 consecutive keys: e4m3 scale from the microblock max / 6
#pragma unroll
          for (int mbk = 0; mbk < 4; ++mbk) {
            float pm = 0.f;
#pragma unroll
            for (int i = 0; i < 16; i += 2)
              pm = fmax3(pm, __uint_as_float(sr[16 * mbk + i]), __uint_as_float(sr[16 * mbk + i + 1]));
            const uint32_t sf = cvt_e4m3x2(0.0f, (pm * kP4Range) * (1.0f / 6.0f)) & 0xffu;
            sfw |= sf << (8 * mbk);
            // 2688 / sf without the SFU: sf = 2^(e-7) (1 + m/8), or m 2^-9 when e = 0
            const uint32_t ex = sf >> 3, mt = sf & 7u;
            const float inv_m = rcp_tab[ex ? mt : 8u + mt];
            const float rr = kP4Range * inv_m * __uint_as_float((ex ? 134u - ex : 136u) << 23);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              uint32_t w = 0;
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const int k = 16 * mbk + 8 * q + 2 * t;
                w |= cvt_e2m1x2(__uint_as_float(sr[k + 1]) * rr, __uint_as_float(sr[k]) * rr) << (8 * t);
              }
              pw[2 * mbk + q] = w;
            }
          }
        }
      }
      if (i8) {
        // INT8 P codes (four per column, key 4i in the low byte) replace this
        // warp's scores in TMEM, where the P·V MMA reads them; the buffer goes
        // back to the score MMAs once that P·V completes
        if (present) tmem_st16(scol, pw);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_FREE + (u & 1)));
      }
      // a rising reference first folds what the phase holds into O (INT8 also
      // every 256 units, before its s32 sums could overflow): the accumulator
      // is settled once the P·V of the unit before completed.  4-bit P goes
      // through shared memory, free once that P·V completed too.
      const bool guard = i8 && u > nu16 && ((u - nu16) & 255) == 0;
      if (!i8 || __any_sync(FULL, raise || guard)) {
        if (!__all_sync(FULL, pfree_wait(u - 1))) return false;
        tc_fence_after();
      }
      fold(raise || guard, i8);
      if (raise) r_lo = r_use;
      l_lo += lp;
      if (present && !i8) {
        {
          uint8_t* pb = smem + SM_P + half * 4096;
#pragma unroll
          for (int c = 0; c < 2; ++c)
            *reinterpret_cast<uint4*>(pb + row * 32 + ((c ^ ((row >> 2) & 1)) * 16)) =
                make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
          *reinterpret_cast<uint32_t*>(smem + SM_P + PO_PSF + half * kSfAtomBytes + (row & 31) * 16 +
                                       (row >> 5) * 4) = sfw;
        }
      }
      if (!i8) fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P_FULL + (u & 1)));
      return true;
    };
    for (int u = nu16; ok && u < nu8; ++u) ok = lowbit_unit(u, std::true_type{});
    for (int u = nu8; ok && u < nu; ++u) ok = lowbit_unit(u, std::false_type{});
    // the last low-bit phase joins O once its last P·V completed
    if (ok && nu > nu16) {
      if (!__all_sync(FULL, pfree_wait(nu - 1))) ok = false;
      tc_fence_after();
      if (ok) fold(true, nu8 == nu);
    }
    if (ok && !__all_sync(FULL, mbar_wait(bar(B_DONE), 0))) ok = false;
    tc_fence_after();
    if (!ok) { raise_timeout(A.status); *abort_flag = 1; }
    // ---- epilogue: O / l in bf16, staged for the TMA store; each warp summed
    // l over its own key blocks, against the reference both warps share
    {
      float* lx = red + 512;
      lx[half * 128 + row] = l16;
      if (!pair_sync(B_EPI + quarter, 0)) { raise_timeout(A.status); *abort_flag = 1; }
      const float lt = l16 + lx[(1 - half) * 128 + row];
      const float il = lt > 0.f ? 1.0f / lt : 0.f;
      uint8_t* ot = smem + SM_Q16 + half * 16384;  // channel half = output sub-tile
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        uint32_t orr[32];
        tmem_ld32(tbase + lane_off + TM_O + half * 64 + c, orr);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(orr[8 * q + 2 * i]) * il,
                                                      __uint_as_float(orr[8 * q + 2 * i + 1]) * il);
            w[i] = *reinterpret_cast<uint32_t*>(&hb);
          }
          const int chunk = (c >> 3) + q;
          *reinterpret_cast<uint4*>(ot + row * 128 + ((chunk ^ (row & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_async_smem();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && !*abort_flag) {
    int cx, cy, cf;
    box(qa, cx, cy, cf);
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                 ::"l"(&tmO), "r"(s0 + SM_Q16), "r"(0), "r"(cx), "r"(cy), "r"(cf) : "memory");
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                 ::"l"(&tmO), "r"(s0 + SM_Q16 + 16384), "r"(64), "r"(cx), "r"(cy), "r"(cf) : "memory");
    if (qb >= 0) {
      box(qb, cx, cy, cf);
      asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                   ::"l"(&tmO), "r"(s0 + SM_Q16 + 8192), "r"(0), "r"(cx), "r"(cy), "r"(cf) : "memory");
      asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                   ::"l"(&tmO), "r"(s0 + SM_Q16 + 16384 + 8192), "r"(64), "r"(cx), "r"(cy), "r"(cf) : "memory");
    }
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    // every issued MMA has completed before the columns are released
    (void)__all_sync(0xffffffffu, mbar_wait(bar(B_DONE), 0));
    tmem_relinquish();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace
}  // namespace da2

// ------------------------------------------------------------------ host side
namespace da2 {
namespace {

// Merged key lists of query-block pairs (2p, 2p+1): per phase (16, 8, 4) the
// ascending key blocks either member keeps in that phase, with member flags and
// a flag for key blocks without padding.
// Per phase, the key blocks either query block of the pair keeps, in the
// order the attention kernel takes them two at a time: ascending, except that
// when the pair has no 16-bit block (so nothing has set the low-bit phases'
// P reference) a low-bit phase takes first the blocks both query blocks keep,
// the likeliest to hold a row's largest scores, so that the reference rises
// early and seldom later; each group ascending.  The two map rows are staged
// in shared memory once for all passes.
__global__ void __launch_bounds__(256) pair_lists_kernel(Geom g, const uint8_t* __restrict__ map,
                                                         uint32_t* __restrict__ plist, int* __restrict__ pcnt,
                                                         int npairs) {
  const int pair = blockIdx.x, bh = blockIdx.y, nb = g.nb;
  const int qa = 2 * pair, qb = (2 * pair + 1 < nb) ? 2 * pair + 1 : -1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  extern __shared__ uint8_t rows_sm[];  // [2][nb]
  {
    const uint8_t* ga = map + ((size_t)bh * nb + qa) * nb;
    const uint8_t* gb = qb >= 0 ? map + ((size_t)bh * nb + qb) * nb : nullptr;
    for (int i = threadIdx.x; i < nb; i += 256) {
      rows_sm[i] = ga[i];
      rows_sm[nb + i] = gb ? gb[i] : (uint8_t)0;
    }
    __syncthreads();
  }
  const uint8_t* ra = rows_sm;
  const uint8_t* rb = qb >= 0 ? rows_sm + nb : nullptr;
  uint32_t* out = plist + ((size_t)bh * npairs + pair) * (2 * nb);
  __shared__ int wtot[3][8];
  __shared__ int tot[3];
  int run = 0;
  int counts[3];
  const int phase_bits[3] = {16, 8, 4};
  for (int ph = 0; ph < 3; ++ph) {
    const int start = run;
    // class of a key block: 0 both keep it, 1 only one of them does
    auto cls = [&](int kb) -> int {
      if (kb >= nb) return -1;
      const bool a = ra[kb] == phase_bits[ph], b = rb && rb[kb] == phase_bits[ph];
      return (a && b && ph > 0 && counts[0] == 0) ? 0 : ((a || b) ? 1 : -1);
    };
    // pass 1 (only when some block can come first): the class sizes
    int n[3] = {0, 0, 0};
    const bool two_groups = ph > 0 && counts[0] == 0;
    for (int base = 0; two_groups && base < nb; base += 256) {
      const int c = cls(base + threadIdx.x);
#pragma unroll
      for (int k = 0; k < 3; ++k) n[k] += __popc(__ballot_sync(0xffffffffu, c == k));
    }
    if (lane == 0) {
#pragma unroll
      for (int k = 0; k < 3; ++k) wtot[k][warp] = n[k];
    }
    __syncthreads();
    if (threadIdx.x < 3) {
      int t = 0;
      for (int w = 0; w < 8; ++w) t += wtot[threadIdx.x][w];
      tot[threadIdx.x] = t;
    }
    __syncthreads();
    const int nc = tot[0];  // the first group's size (0 for one ascending group)
    __syncthreads();
    // pass 2: each entry at its place
    int seen[3] = {0, 0, 0};  // entries of each class before this chunk
    for (int base = 0; base < nb; base += 256) {
      const int kb = base + threadIdx.x;
      const int c = cls(kb);
      unsigned bal[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) bal[k] = __ballot_sync(0xffffffffu, c == k);
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < 3; ++k) wtot[k][warp] = __popc(bal[k]);
      }
      __syncthreads();
      if (c >= 0) {
        int i = seen[c] + __popc(bal[c] & ((1u << lane) - 1u));  // rank within the class
        for (int w = 0; w < warp; ++w) i += wtot[c][w];
        const int off = c == 0 ? i : nc + i;
        const int rx = kb % g.nrx, ry = (kb / g.nrx) % g.nry;
        const bool full = (ry + 1) * g.rh <= g.Hh && (rx + 1) * g.rw <= g.Ww;
        const bool a = ra[kb] == phase_bits[ph], b = rb && rb[kb] == phase_bits[ph];
        out[start + off] = (uint32_t)kb | ((uint32_t)a << 16) | ((uint32_t)b << 17) | ((uint32_t)ph << 18) |
                           ((uint32_t)full << 20);
      }
#pragma unroll
      for (int k = 0; k < 3; ++k)
        for (int w = 0; w < 8; ++w) seen[k] += wtot[k][w];
      __syncthreads();
    }
    run = start + seen[0] + seen[1];
    counts[ph] = run - start;
  }
  if (threadIdx.x == 0)
    *reinterpret_cast<int4*>(pcnt + ((size_t)bh * npairs + pair) * 4) = make_int4(counts[0], counts[1], counts[2], 0);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B*H*T frames][Hh][Ww][d] bf16 view of a [B,H,N,d] tensor, 64-channel x region boxes.
bool map_regions(CUtensorMap* m, const void* base, const Geom& g) {
  const cuuint64_t dims[4] = {(cuuint64_t)g.d, (cuuint64_t)g.Ww, (cuuint64_t)g.Hh, (cuuint64_t)g.BH * g.T};
  const cuuint64_t strides[3] = {(cuuint64_t)g.d * 2, (cuuint64_t)g.Ww * g.d * 2, (cuuint64_t)g.Hh * g.Ww * g.d * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)g.rw, (cuuint32_t)g.rh, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major byte matrix [rows][rowbytes] in boxes of box_rows rows.
bool map_rows(CUtensorMap* m, const void* base, uint64_t rows, uint32_t rowbytes, uint32_t box_rows,
              CUtensorMapSwizzle sw) {
  const cuuint64_t dims[2] = {rowbytes, rows};
  const cuuint64_t strides[1] = {rowbytes};
  const cuuint32_t box[2] = {rowbytes, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tma_available() { return encode_fn() != nullptr; }

bool make_region_map(CUtensorMap* m, const void* base, const Geom& g, bool swizzle128) {
  const cuuint64_t dims[4] = {(cuuint64_t)g.d, (cuuint64_t)g.Ww, (cuuint64_t)g.Hh, (cuuint64_t)g.BH * g.T};
  const cuuint64_t strides[3] = {(cuuint64_t)g.d * 2, (cuuint64_t)g.Ww * g.d * 2, (cuuint64_t)g.Hh * g.Ww * g.d * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)g.rw, (cuuint32_t)g.rh, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return encode_fn() && encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool attention_tc_supported(const Geom& g) {
  return g.d == kD && g.BH <= 65535 && encode_fn() != nullptr;
}

// Status word of the dense path (its waits are bounded like the sparse path's;
// the dense entry point has no workspace to report through).
__device__ int g_dense_status;

bool dense_tc_supported(int B, int H, int N, int d) {
  return d == kD && N >= 64 && (long long)B * H <= 65535 && encode_fn() != nullptr;
}

// Dense attention on the same kernel: the token axis viewed as one frame of
// 1 x N tokens cut into 64-token regions (natural order), every key block in
// the 16-bit phase, the tail block masked and clipped by TMA like a padded region.
cudaError_t launch_dense_tc(int B, int H, int N, const void* q, const void* k, const void* v, void* out,
                            cudaStream_t st) {
  Geom g{};
  g.B = B; g.H = H; g.T = 1; g.Hh = 1; g.Ww = N; g.d = kD; g.rh = 1; g.rw = 64;
  g.nry = 1; g.nrx = (N + 63) / 64; g.nb = g.nrx; g.N = N; g.BH = B * H;
  CUtensorMap tq, tk, tv, to;
  if (!map_regions(&tq, q, g) || !map_regions(&tk, k, g) || !map_regions(&tv, v, g) || !map_regions(&to, out, g))
    return cudaErrorInvalidValue;
  int* status = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_dense_status);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(status, 0, sizeof(int), st)) != cudaSuccess) return e;
  TcArgs A{};
  A.status = status;
  A.npairs = (g.nb + 1) / 2;
  e = cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  // the low-bit tensor maps are never used in dense mode
  attn_tc_kernel<true><<<dim3(A.npairs, g.BH), kThreads, kSmemBytes, st>>>(tq, tk, tv, to, tq, tk, tv, tq, tk, tv, g, A);
  return cudaGetLastError();
}

cudaError_t launch_pair_lists(const Geom& g, const Layout& L, void* ws, cudaStream_t st) {
  const int npairs = (g.nb + 1) / 2;
  const size_t smem = (2 * (size_t)g.nb + 15) & ~(size_t)15;  // the pair's two map rows
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(pair_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  pair_lists_kernel<<<dim3(npairs, g.BH), 256, smem, st>>>(g, at<uint8_t>(ws, L, R_MAP), at<uint32_t>(ws, L, R_PLIST),
                                                          at<int>(ws, L, R_PCNT), npairs);
  return cudaGetLastError();
}

cudaError_t launch_attention_tc(const Geom& g, const Layout& L, const void* q, const void* k, const void* v,
                                void* ws, void* out, cudaStream_t st) {
  CUtensorMap tq, tk, tv, to, tq8, tk8, tv8, tq4, tk4, tv4;
  const uint64_t rows64 = (uint64_t)g.BH * g.nb * 64, rows128 = (uint64_t)g.BH * g.nb * kD;
  if (!map_regions(&tq, q, g) || !map_regions(&tk, k, g) || !map_regions(&tv, v, g) || !map_regions(&to, out, g) ||
      !map_rows(&tq8, at<int8_t>(ws, L, R_Q_I8), rows64, kD, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map_rows(&tk8, at<int8_t>(ws, L, R_K_I8), rows64, kD, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map_rows(&tv8, at<int8_t>(ws, L, R_V_I8), rows128, 64, kD, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !map_rows(&tq4, at<uint8_t>(ws, L, R_Q_F4), rows64, kD / 2, 64, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !map_rows(&tk4, at<uint8_t>(ws, L, R_K_F4), rows64, kD / 2, 64, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !map_rows(&tv4, at<uint8_t>(ws, L, R_V_F4), rows128, 32, kD, CU_TENSOR_MAP_SWIZZLE_32B))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_pair_lists(g, L, ws, st);
  if (e != cudaSuccess) return e;
  int* status = at<int>(ws, L, R_STATUS);
  TcArgs A;
  A.plist = at<uint32_t>(ws, L, R_PLIST);
  A.pcnt = at<int>(ws, L, R_PCNT);
  A.q_s8 = at<float>(ws, L, R_Q_S8);
  A.k_s8 = at<float>(ws, L, R_K_S8);
  A.v_s8 = at<float>(ws, L, R_V_S8);
  A.v_g4 = at<float>(ws, L, R_V_G4);
  A.q_sf4 = at<uint8_t>(ws, L, R_Q_SF4);
  A.k_sf4 = at<uint8_t>(ws, L, R_K_SF4);
  A.v_sf4 = at<uint8_t>(ws, L, R_V_SF4);
  A.status = status;
  A.npairs = (g.nb + 1) / 2;
  e = cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<false><<<dim3(A.npairs, g.BH), kThreads, kSmemBytes, st>>>(tq, tk, tv, to, tq8, tk8, tv8, tq4, tk4,
                                                                             tv4, g, A);
  return cudaGetLastError();
}

}  // namespace da2
