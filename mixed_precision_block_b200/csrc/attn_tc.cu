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
// Roles (10 warps): warps 0-7 softmax — warp w owns TMEM lanes 32(w&3).. (tile
// rows) and half h = w>>2 of every key block (keys 32h..32h+31) and of the
// channels (64h..64h+63); warp 8 issues TMA loads; warp 9 issues the MMAs from
// a non-blocking scheduler that starts S of a block as soon as its buffers are
// free, ahead of the P·V of the block before.
//   16-bit  S = Q·K^T (kind::f16 bf16, M128 N64, fp32 TMEM, 2 buffers);
//           P = exp2(s·log2e/√d − m_ref) rounded to bf16, m_ref an integer
//           exponent raised lazily (O rescaled in TMEM by a power of two only
//           when the row max grows by more than 2^8); P goes K-major to shared
//           memory; O += P·V (kind::f16, V read MN-major from the TMA tile).
//   8-bit   S = Q8·K8^T (kind::i8, s32); P8 = round(255·exp(s − m_blk)) as u8;
//           X = P8·V8^T (kind::i8 u8×s8, s32, 2 buffers); each softmax warp
//           folds its 64 channels of X into a register accumulator weighted by
//           exp(m_blk − m8); the per-channel V scale is applied once, at the
//           phase boundary, when the register accumulator joins O.
//   4-bit   S = Q4·K4^T (kind::mxf4nvf4, block16 e4m3 scales copied into TMEM
//           with tcgen05.cp from the scale atoms prep wrote); P re-quantised to
//           NVFP4 per 16 keys in registers, with its scales written as an atom;
//           X = P4·V4^T (block-scaled, fp32), folded into the register
//           accumulator; the channel scale g is applied at the end.  Entering
//           the phase, the INT8 accumulator is folded into O with its own
//           channel scale first — the phase-boundary rescale.
// Operands arrive by TMA: bf16 Q/K/V as 8×8-token region boxes straight from
// the [B,H,N,d] tensors (padding is the TMA zero fill), INT8 codes as 2-D
// boxes of the workspace.  The epilogue writes O through the same region box
// with a TMA store, whose clipping drops the padding rows — the restore.
// Every mbarrier wait is bounded; on expiry the CTA raises the workspace status
// word, skips the rest and releases its tensor memory.
#include <cuda.h>

#include <mutex>

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

// shared-memory map (offsets from a 1024-aligned base)
constexpr uint32_t SM_Q16 = 0;         // [2 halves][128 rows][128 B], SW128
constexpr uint32_t SM_Q8 = 32768;      // [128 rows][128 B], SW128
constexpr uint32_t SM_K = 49152;       // K ring: kStages x 32 KB
constexpr uint32_t SM_V = SM_K + kStages * 32768;            // V ring: kStages x 32 KB
// 16-bit unit (key blocks a, b): K slot = K_a h0 | K_b h0 | K_a h1 | K_b h1 (8 KB
// each, so each channel half of [K_a; K_b] is one 128-row K-major operand);
// V slot = V_a | V_b (16 KB each).  INT8 unit (one key block): K8 (8 KB), V8^T (8 KB).
constexpr uint32_t SM_P = SM_V + kStages * 32768;            // P_a | P_b, 16 KB each
constexpr uint32_t SM_VS = SM_P + 32768;                     // V channel scales: INT8 | NVFP4 g (fp32)
constexpr uint32_t SM_RED = SM_VS + 1024;                    // row-statistics exchange, 4 KB
constexpr uint32_t SM_BAR = SM_RED + 4096;                   // mbarriers
constexpr uint32_t SM_MISC = SM_BAR + 512;
constexpr uint32_t SM_PSF = SM_MISC + 128;                   // scale atom of the 4-bit P (512 B)
constexpr uint32_t SM_Q4 = (SM_PSF + 512 + 1023) & ~1023u;   // NVFP4 Q of the pair [128][64 B], SW64
constexpr uint32_t SM_TOTAL = SM_Q4 + 8192;
// 4-bit unit: K slot = K4 [64][64 B] SW64 at +0, its scale atoms (2 x 512 B) at
// +8192; V slot = V4^T [128][32 B] SW32 at +0, its scale atom at +8192
constexpr uint32_t SL_SF = 8192;
constexpr uint32_t kSmemBytes = SM_TOTAL + 1024;  // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// TMEM columns: O 0-127, S 2 x 128 at 128 (a 16-bit unit fills 128, an INT8 or
// 4-bit unit 64), X 128 at 384.  4-bit units keep their scale factors in the
// upper half of their S buffer: K scales at +64, V scales at +72, P scales at
// +76; Q's scales (constant for the CTA) at 216.  Scale columns are 4-aligned.
constexpr uint32_t TM_O = 0, TM_S = 128, TM_X = 384;
constexpr uint32_t TM_SFQ = 216, TMO_SFK = 64, TMO_SFV = 72, TMO_SFP = 76;

// mbarrier slots (8 bytes each)
enum {
  B_Q16 = 0, B_Q8, B_Q4, B_SFQ, B_K_FULL, B_K_EMPTY = B_K_FULL + kStages, B_V_FULL = B_K_EMPTY + kStages,
  B_V_EMPTY = B_V_FULL + kStages, B_S_FULL = B_V_EMPTY + kStages,
  B_S_FREE = B_S_FULL + 2, B_P_FULL = B_S_FREE + 2, B_P_FREE = B_P_FULL + 1, B_X_FULL = B_P_FREE + 1,
  B_X_FREE = B_X_FULL + 1, B_DONE = B_X_FREE + 1,
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

// Exact int32 -> fp32 for |x| < 2^22 on the integer and FMA pipes (the I2F
// conversion unit is a narrow pipe): 1.5*2^23 + x has x in its low mantissa bits.
__device__ __forceinline__ float i2f_small(uint32_t x) {
  return __int_as_float((int)x + 0x4B400000) - 12582912.0f;
}
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
// round-to-nearest-even of a value in [0, 2^22) to an integer in the low bits,
// again through the mantissa of 1.5*2^23 (the add rounds ties to even)
__device__ __forceinline__ uint32_t rne_small(float v) {
  return (uint32_t)__float_as_int(v + 12582912.0f) & 0x3FFFFFu;
}

// Items: kb | inA << 16 | inB << 17 | kind << 18 (kind 0 = 16-bit, 1 = 8-bit)
//        | full << 20 (the key block has no padding slot).
__device__ __forceinline__ int item_kb(uint32_t e) { return (int)(e & 0xffffu); }
__device__ __forceinline__ int item_kind(uint32_t e) { return (int)((e >> 18) & 3u); }

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

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const __grid_constant__ CUtensorMap tmQ8, const __grid_constant__ CUtensorMap tmK8,
               const __grid_constant__ CUtensorMap tmV8, const __grid_constant__ CUtensorMap tmQ4,
               const __grid_constant__ CUtensorMap tmK4, const __grid_constant__ CUtensorMap tmV4, Geom g,
               TcArgs A) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s0 = (uint32_t)__cvta_generic_to_shared(smem);
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qa = 2 * pair, qb = (2 * pair + 1 < g.nb) ? 2 * pair + 1 : -1;
  const size_t prow = (size_t)bh * A.npairs + pair;
  const int4 pc = *reinterpret_cast<const int4*>(A.pcnt + prow * 4);
  const int n16 = pc.x, n8 = pc.y, n4 = pc.z;
  const uint32_t* items = A.plist + prow * (size_t)(2 * g.nb);
  auto bar = [&](int i) { return s0 + SM_BAR + 8u * (uint32_t)i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + SM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM_MISC + 8);

  // units: 16-bit items are taken two at a time (one N = 128 score MMA per
  // unit), INT8 items one at a time
  const int nu16 = (n16 + 1) / 2;
  const int nu8 = nu16 + n8;  // INT8 units end here, 4-bit units follow
  const int nu = nu8 + n4;
  auto unit_items = [&](int u, int& i0, int& cnt) {
    if (u < nu16) { i0 = 2 * u; cnt = min(2, n16 - 2 * u); }
    else { i0 = n16 + (u - nu16); cnt = 1; }  // INT8 and 4-bit items follow in list order
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
    mbar_init(bar(B_P_FULL), kSoftmaxWarps);
    mbar_init(bar(B_P_FREE), 1);
    mbar_init(bar(B_X_FULL), 1);
    mbar_init(bar(B_X_FREE), kSoftmaxWarps);
    mbar_init(bar(B_DONE), 1);
    for (int i = 0; i < 8; ++i) mbar_init(bar(B_PAIR + i), 2);
    for (int i = 0; i < 4; ++i) mbar_init(bar(B_EPI + i), 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(s0 + SM_MISC, 512);
  if (threadIdx.x < kD) {
    reinterpret_cast<float*>(smem + SM_VS)[threadIdx.x] = A.v_s8[(size_t)bh * kD + threadIdx.x];
    reinterpret_cast<float*>(smem + SM_VS + 512)[threadIdx.x] = A.v_g4[(size_t)bh * kD + threadIdx.x];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];

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
              box(item_kb(items[i0 + t]), cx, cy, cf);
              tma_load_4d(dst + t * 8192, &tmK, fb, 0, cx, cy, cf);
              tma_load_4d(dst + 16384 + t * 8192, &tmK, fb, 64, cx, cy, cf);
            }
          } else if (kn < nu8) {
            mbar_expect_tx(fb, 8192u);
            tma_load_2d(dst, &tmK8, fb, 0, (bh * g.nb + item_kb(items[i0])) * 64);
          } else {
            const size_t kl = (size_t)bh * g.nb + item_kb(items[i0]);
            mbar_expect_tx(fb, 4096u + 1024u);
            tma_load_2d(dst, &tmK4, fb, 0, (int)(kl * 64));
            bulk_load(dst + SL_SF, A.k_sf4 + kl * 2 * kSfAtomBytes, 2 * kSfAtomBytes, fb);
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
              box(item_kb(items[i0 + t]), cx, cy, cf);
              tma_load_4d(dst + t * 16384, &tmV, fb, 0, cx, cy, cf);
              tma_load_4d(dst + t * 16384 + 8192, &tmV, fb, 64, cx, cy, cf);
            }
          } else if (vn < nu8) {
            mbar_expect_tx(fb, 8192u);
            tma_load_2d(dst, &tmV8, fb, 0, (bh * g.nb + item_kb(items[i0])) * kD);
          } else {
            const size_t kl = (size_t)bh * g.nb + item_kb(items[i0]);
            mbar_expect_tx(fb, 4096u + kSfAtomBytes);
            tma_load_2d(dst, &tmV4, fb, 0, (int)(kl * kD));
            bulk_load(dst + SL_SF, A.v_sf4 + kl * kSfAtomBytes, kSfAtomBytes, fb);
          }
          ++vn;
          progressed = true;
        }
        if (progressed) {
          idle = 0;
        } else if (++idle > (1u << 26) || *abort_flag) {
          raise_timeout(A.status); *abort_flag = 1;
          break;
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA scheduler
    if (elect_one()) {
      const uint32_t id16n128 = idesc(kDF32, kFmtBF16, kFmtBF16, false, false, 128, 128);
      const uint32_t id16n64 = idesc(kDF32, kFmtBF16, kFmtBF16, false, false, 128, 64);
      const uint32_t idpv = idesc(kDF32, kFmtBF16, kFmtBF16, false, true, 128, 128);
      const uint32_t id8 = idesc(kDS32, kFmtS8, kFmtS8, false, false, 128, 64);
      const uint32_t idx8 = idesc(kDS32, kFmtU8, kFmtS8, false, false, 128, 128);
      const uint32_t id4s = idesc_f4(128, 64), id4pv = idesc_f4(128, 128);
      bool f4_ready = false;  // Q4 loaded and its scales in TMEM
      bool ok = true;
      if (n16 > 0) ok = ok && mbar_wait(bar(B_Q16), 0);
      if (n8 > 0) ok = ok && mbar_wait(bar(B_Q8), 0);
      int sn = 0, pn = 0, xu = 0;  // next unit for S, next unit for P·V, INT8 results issued
      uint32_t idle = 0;
      while (ok && pn < nu) {
        bool progressed = false;
        if (sn < nu) {
          const int s = sn % kStages, b = sn & 1;
          if (sn >= nu8 && !f4_ready) {
            // first 4-bit unit: Q4 must be in shared memory and its scales in TMEM
            f4_ready = mbar_test(bar(B_Q4), 0) && mbar_test(bar(B_SFQ), 0);
          }
          if ((sn < nu8 || f4_ready) && mbar_test(bar(B_K_FULL + s), (sn / kStages) & 1) &&
              (sn < 2 || mbar_test(bar(B_S_FREE + b), ((sn >> 1) - 1) & 1))) {
            tc_fence_after();
            const uint32_t st = s0 + SM_K + s * 32768;
            const uint32_t sd = tbase + TM_S + b * 128;
            if (sn < nu16) {
              int i0, cnt;
              unit_items(sn, i0, cnt);
              const uint32_t id = cnt == 2 ? id16n128 : id16n64;
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int h = k >> 2, kk = k & 3;
                mma_f16(sd, smem_desc(s0 + SM_Q16 + h * 16384 + kk * 32, 16, 1024, SW_128),
                        smem_desc(st + h * 16384 + kk * 32, 16, 1024, SW_128), id, k > 0 ? 1u : 0u);
              }
            } else if (sn < nu8) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_i8(sd, smem_desc(s0 + SM_Q8 + kk * 32, 16, 1024, SW_128),
                       smem_desc(st + kk * 32, 16, 1024, SW_128), id8, kk > 0 ? 1u : 0u);
            } else {
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                tc_cp_atom(sd + TMO_SFK + 4 * c, st + SL_SF + c * kSfAtomBytes);
                mma_f4(sd, smem_desc(s0 + SM_Q4 + 32 * c, 16, 512, SW_64), smem_desc(st + 32 * c, 16, 512, SW_64),
                       id4s, c > 0 ? 1u : 0u, tbase + TM_SFQ + 4 * c, sd + TMO_SFK + 4 * c);
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
          const bool int8 = pn >= nu16;  // INT8 or 4-bit: both produce a block result X
          if (mbar_test(bar(B_V_FULL + s), (pn / kStages) & 1) && mbar_test(bar(B_P_FULL), pn & 1) &&
              (!int8 || xu < 1 || mbar_test(bar(B_X_FREE), (xu - 1) & 1))) {
            tc_fence_after();
            const uint32_t st = s0 + SM_V + s * 32768;
            const uint32_t pbuf = s0 + SM_P;
            if (!int8) {
              int i0, cnt;
              unit_items(pn, i0, cnt);
              for (int t = 0; t < cnt; ++t) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_f16(tbase + TM_O, smem_desc(pbuf + t * 16384 + kk * 32, 16, 1024, SW_128),
                          smem_desc(st + t * 16384 + kk * 2048, 8192, 1024, SW_128), idpv, 1u);
              }
            } else if (pn < nu8) {
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                mma_i8(tbase + TM_X, smem_desc(pbuf + kk * 32, 16, 512, SW_64),
                       smem_desc(st + kk * 32, 16, 512, SW_64), idx8, kk > 0 ? 1u : 0u);
              mma_commit(bar(B_X_FULL));
              ++xu;
            } else {
              const uint32_t sfb = tbase + TM_S + (pn & 1) * 128;
              tc_cp_atom(sfb + TMO_SFV, st + SL_SF);
              tc_cp_atom(sfb + TMO_SFP, s0 + SM_PSF);
              mma_f4(tbase + TM_X, smem_desc(pbuf, 16, 256, SW_32), smem_desc(st, 16, 256, SW_32), id4pv, 0u,
                     sfb + TMO_SFP, sfb + TMO_SFV);
              mma_commit(bar(B_X_FULL));
              ++xu;
            }
            mma_commit(bar(B_P_FREE));
            mma_commit(bar(B_V_EMPTY + s));
            ++pn;
            progressed = true;
          }
        }
        if (progressed) {
          idle = 0;
        } else if (++idle > (1u << 26) || *abort_flag) {
          ok = false;
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
    const float* vs = reinterpret_cast<const float*>(smem + SM_VS);
    float* red = reinterpret_cast<float*>(smem + SM_RED);  // [2][2][128]
    const unsigned FULL = 0xffffffffu;
    // the two warps of a row quarter exchange row statistics through shared
    // memory, ordered by an mbarrier (bounded wait, unlike a named barrier)
    auto pair_sync = [&](int idx, uint32_t parity) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(idx));
      return __all_sync(FULL, mbar_wait(bar(idx), parity));
    };
    float m16 = -INFINITY, l16 = 0.f;  // 16-bit phase: O in TMEM, integer reference
    float m8 = -INFINITY, l8 = 0.f;    // 8-bit phase: register accumulator
    bool ok = true;
    {  // O starts at zero (this warp's 64 columns)
      uint32_t z[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = 0u;
      tmem_st32(tbase + lane_off + TM_O + half * 64, z);
      tmem_st32(tbase + lane_off + TM_O + half * 64 + 32, z);
      tmem_wait_st();
    }
    for (int u = 0; ok && u < nu16; ++u) {
      if (__any_sync(FULL, *abort_flag != 0)) { ok = false; break; }
      const int b = u & 1;
      int i0, cnt;
      unit_items(u, i0, cnt);
      float* xch = red + (u & 1) * 256;  // [2 halves][128 rows] for this unit
      const uint32_t sbase = tbase + lane_off + TM_S + b * 128;
      if (!__all_sync(FULL, mbar_wait(bar(B_S_FULL + b), (u >> 1) & 1))) { ok = false; break; }
      tc_fence_after();
        // ---- 16-bit unit: this warp owns key block `half` of the unit
        const bool present = half < cnt;
        const uint32_t e = present ? items[i0 + half] : 0u;
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
        mx = fmaxf(mx, xch[(1 - half) * 128 + row]) * sl2;  // unit row max, log2 units
        const bool row_live = mx != -INFINITY;  // the row is a member of some block of the unit
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
        // the P buffer and O are free once the P·V of unit u-1 completed
        if (!__all_sync(FULL, u < 1 || mbar_wait(bar(B_P_FREE), (u - 1) & 1))) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(FULL, need_o)) {
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
        if (present) {
          uint8_t* pb = smem + SM_P + half * 16384;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(pb + row * 128 + ((c ^ (row & 7)) * 16)) =
                make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
        }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P_FULL));
    }
    // the INT8 register accumulator lives only through the 8-bit phase
    float o8[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) o8[i] = 0.f;
    int xu = 0;
    bool have_pend = false, pend_member = false;
    float pend_mb = 0.f, pend_lb = 0.f;
    // fold the X of the pending INT8 item into the register accumulator
    auto merge_x = [&]() -> bool {
      if (!__all_sync(FULL, mbar_wait(bar(B_X_FULL), xu & 1))) return false;
      tc_fence_after();
      if (pend_member) {
        uint32_t xr[64];
        tmem_ld32(tbase + lane_off + TM_X + half * 64, xr);
        tmem_ld32(tbase + lane_off + TM_X + half * 64 + 32, xr + 32);
        tmem_wait_ld();
        if (pend_mb > m8 + kRescaleThreshold || m8 == -INFINITY) {
          const float nm = ceilf(pend_mb);
          const float a = (m8 == -INFINITY) ? 0.f : ldexpf(1.0f, (int)(m8 - nm));
#pragma unroll
          for (int i = 0; i < 64; ++i) o8[i] *= a;
          l8 *= a;
          m8 = nm;
        }
        const float w = fast_exp2(pend_mb - m8);
        const float f = w * (1.0f / 255.0f);
        l8 += pend_lb * w;
        const uint64_t fx2 = f2pack(f, f), kx2 = f2pack(-12582912.0f, -12582912.0f);
#pragma unroll
        for (int i = 0; i < 64; i += 2) {  // |X| < 64*255*127 < 2^22: exact through the mantissa
          const uint64_t xf = f2add(f2pack(__int_as_float((int)xr[i] + 0x4B400000),
                                           __int_as_float((int)xr[i + 1] + 0x4B400000)), kx2);
          f2unpack(f2fma(fx2, xf, f2pack(o8[i], o8[i + 1])), o8[i], o8[i + 1]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_X_FREE));
      ++xu;
      have_pend = false;
      return true;
    };

    for (int u = nu16; ok && u < nu8; ++u) {
      if (__any_sync(FULL, *abort_flag != 0)) { ok = false; break; }
      const int b = u & 1;
      int i0, cnt;
      unit_items(u, i0, cnt);
      float* xch = red + (u & 1) * 256;  // [2 halves][128 rows] for this unit
      const uint32_t sbase = tbase + lane_off + TM_S + b * 128;
      // ---- INT8 unit: one key block; this warp owns keys 32*half..+31
      const uint32_t e = items[i0];
      const int kb = item_kb(e);
      const float sk = A.k_s8[(size_t)bh * g.nb + kb];  // issued before the wait
      if (!__all_sync(FULL, mbar_wait(bar(B_S_FULL + b), (u >> 1) & 1))) { ok = false; break; }
      tc_fence_after();
        const bool member = ((e >> (in_b ? 17 : 16)) & 1u) != 0;
        uint32_t sr[32];
        tmem_ld32(sbase + half * 32, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_FREE + b));
        const unsigned long long vm = item_full(e) ? ~0ull : (key_mask(g, kb) >> (32 * half));
        const bool full = (uint32_t)vm == 0xffffffffu;
        int imx = INT_MIN;
        if (member) {
          if (!full) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (!((vm >> i) & 1ull)) sr[i] = (uint32_t)INT_MIN;
          }
          int i4[4] = {INT_MIN, INT_MIN, INT_MIN, INT_MIN};
#pragma unroll
          for (int i = 0; i < 32; ++i) i4[i & 3] = max(i4[i & 3], (int)sr[i]);
          imx = max(max(i4[0], i4[1]), max(i4[2], i4[3]));
        }
        reinterpret_cast<int*>(xch)[half * 128 + row] = imx;
        if (!pair_sync(B_PAIR + quarter * 2 + (u & 1), (u >> 1) & 1)) { ok = false; break; }
        imx = max(imx, reinterpret_cast<const int*>(xch)[(1 - half) * 128 + row]);
        float mb = -INFINITY, lb = 0.f;
        uint32_t pw[8];
        if (member) {
          const float sc = sq * sk * sl2;
          mb = i2f_small((uint32_t)imx) * sc;  // sc >= 0: the max of the scores; |S| < 128*127^2 < 2^22
          const uint64_t scx2 = f2pack(sc, sc), negm = f2pack(-mb, -mb);
          const uint64_t kx2 = f2pack(-12582912.0f, -12582912.0f);
          const uint64_t c255 = f2pack(255.0f, 255.0f), kmag = f2pack(12582912.0f, 12582912.0f);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            uint32_t c[4];
#pragma unroll
            for (int q = 0; q < 4; q += 2) {
              const int k = 4 * i + q;
              // exact int -> float through the mantissa of 1.5*2^23, then the score
              const uint64_t sf = f2add(f2pack(__int_as_float((int)sr[k] + 0x4B400000),
                                               __int_as_float((int)sr[k + 1] + 0x4B400000)), kx2);
              float x0, x1;
              f2unpack(f2fma(sf, scx2, negm), x0, x1);
              float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
              if (!full) {  // padding keys contribute nothing, whatever the block scale
                if (!((vm >> k) & 1ull)) p0 = 0.f;
                if (!((vm >> (k + 1)) & 1ull)) p1 = 0.f;
              }
              const uint64_t pp = f2pack(p0, p1);
              acc[(i * 2 + (q >> 1)) & 3] = f2add(acc[(i * 2 + (q >> 1)) & 3], pp);
              float r0, r1;  // 255 p + 1.5*2^23: round-to-nearest-even code in the low byte
              f2unpack(f2fma(pp, c255, kmag), r0, r1);
              c[q] = __float_as_uint(r0);
              c[q + 1] = __float_as_uint(r1);
            }
            pw[i] = pack_low_bytes(c[0], c[1], c[2], c[3]);
          }
          float s0, s1, s2, s3;
          f2unpack(f2add(acc[0], acc[1]), s0, s1);
          f2unpack(f2add(acc[2], acc[3]), s2, s3);
          lb = (s0 + s1) + (s2 + s3);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) pw[i] = 0u;
        }
        if (!__all_sync(FULL, u < 1 || mbar_wait(bar(B_P_FREE), (u - 1) & 1))) { ok = false; break; }
        uint8_t* pb = smem + SM_P;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int chunk = half * 2 + c;
          *reinterpret_cast<uint4*>(pb + row * 64 + ((chunk ^ ((row >> 1) & 3)) * 16)) =
              make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
        }
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_P_FULL));
        if (have_pend && !merge_x()) { ok = false; break; }
        have_pend = true;
        pend_member = member;
        pend_mb = mb;
        pend_lb = lb;
    }
    if (ok && have_pend) ok = merge_x();
    const float* vsc = reinterpret_cast<const float*>(smem + SM_VS);  // scale of the register accumulator
    if (ok && n4 > 0) {
      // ---- phase boundary 8 -> 4: fold the INT8 accumulator into O with its
      // channel scale, so the registers can carry the 4-bit phase
      if (n8 > 0) {
        const float mm = fmaxf(m16, m8);
        const float a16 = m16 == -INFINITY ? 0.f : fast_exp2(m16 - mm);
        const float a8 = m8 == -INFINITY ? 0.f : fast_exp2(m8 - mm);
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          uint32_t orr[32];
          tmem_ld32(tbase + lane_off + TM_O + half * 64 + c, orr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            orr[i] = __float_as_uint(a16 * __uint_as_float(orr[i]) + a8 * vs[half * 64 + c + i] * o8[c + i]);
          tmem_st32(tbase + lane_off + TM_O + half * 64 + c, orr);
        }
        tmem_wait_st();
        l16 = l16 * a16 + l8 * a8;
        m16 = mm;
#pragma unroll
        for (int i = 0; i < 64; ++i) o8[i] = 0.f;
        m8 = -INFINITY;
        l8 = 0.f;
      }
      // Q's scale factors into TMEM (each lane quarter holds all 128 rows)
      if (half == 0) {
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
      vsc = reinterpret_cast<const float*>(smem + SM_VS + 512);  // g
      // fold a 4-bit block result X (fp32) into the register accumulator
      auto merge_x4 = [&]() -> bool {
        if (!__all_sync(FULL, mbar_wait(bar(B_X_FULL), xu & 1))) return false;
        tc_fence_after();
        if (pend_member) {
          uint32_t xr[64];
          tmem_ld32(tbase + lane_off + TM_X + half * 64, xr);
          tmem_ld32(tbase + lane_off + TM_X + half * 64 + 32, xr + 32);
          tmem_wait_ld();
          if (pend_mb > m8 + kRescaleThreshold || m8 == -INFINITY) {
            const float nm = ceilf(pend_mb);
            const float a = (m8 == -INFINITY) ? 0.f : ldexpf(1.0f, (int)(m8 - nm));
#pragma unroll
            for (int i = 0; i < 64; ++i) o8[i] *= a;
            l8 *= a;
            m8 = nm;
          }
          const float f = fast_exp2(pend_mb - m8);
          l8 += pend_lb * f;
          const uint64_t fx2 = f2pack(f, f);
#pragma unroll
          for (int i = 0; i < 64; i += 2)
            f2unpack(f2fma(fx2, f2pack(__uint_as_float(xr[i]), __uint_as_float(xr[i + 1])), f2pack(o8[i], o8[i + 1])),
                     o8[i], o8[i + 1]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_X_FREE));
        ++xu;
        have_pend = false;
        return true;
      };
      for (int u = nu8; ok && u < nu; ++u) {
        if (__any_sync(FULL, *abort_flag != 0)) { ok = false; break; }
        const int b = u & 1;
        int i0, cnt;
        unit_items(u, i0, cnt);
        float* xch = red + (u & 1) * 256;
        const uint32_t sbase = tbase + lane_off + TM_S + b * 128;
        // ---- 4-bit unit: one key block; this warp owns keys 32*half..+31
        const uint32_t e = items[i0];
        const int kb = item_kb(e);
        const bool member = ((e >> (in_b ? 17 : 16)) & 1u) != 0;
        if (!__all_sync(FULL, mbar_wait(bar(B_S_FULL + b), (u >> 1) & 1))) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[32];
        tmem_ld32(sbase + half * 32, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_FREE + b));
        const unsigned long long vm = item_full(e) ? ~0ull : (key_mask(g, kb) >> (32 * half));
        const bool full = (uint32_t)vm == 0xffffffffu;
        float mx = -INFINITY;
        if (member) {
          if (!full) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (!((vm >> i) & 1ull)) sr[i] = __float_as_uint(-INFINITY);
          }
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int i = 0; i < 32; i += 8)
#pragma unroll
            for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], __uint_as_float(sr[i + 2 * q]), __uint_as_float(sr[i + 2 * q + 1]));
          mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
        }
        xch[half * 128 + row] = mx;
        if (!pair_sync(B_PAIR + quarter * 2 + (u & 1), (u >> 1) & 1)) { ok = false; break; }
        mx = fmaxf(mx, xch[(1 - half) * 128 + row]);
        float mb = -INFINITY, lb = 0.f;
        uint32_t pw[4] = {0u, 0u, 0u, 0u};
        uint32_t sfw = 0u;  // this half-row's two e4m3 P scales
        if (member) {
          mb = mx * sl2;
          float pv[32];
          const uint64_t sl2x2 = f2pack(sl2, sl2), negm = f2pack(-mb, -mb);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1;
            f2unpack(f2fma(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), sl2x2, negm), x0, x1);
            pv[2 * i] = fast_exp2(x0);
            pv[2 * i + 1] = fast_exp2(x1);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) lb += pv[i];
          // NVFP4 over 16 consecutive keys: e4m3 scale from the microblock max / 6
#pragma unroll
          for (int mbk = 0; mbk < 2; ++mbk) {
            float pm = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) pm = fmaxf(pm, pv[16 * mbk + i]);
            const uint32_t sf = cvt_e4m3x2(0.0f, __fdiv_rn(pm, 6.0f)) & 0xffu;
            sfw |= sf << (8 * mbk);
            const float dec = e4m3_to_f32(sf);
            if (dec != 0.f) {
              const float r = __fdiv_rn(1.0f, dec);
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                uint32_t w = 0;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                  const int k = 16 * mbk + 8 * q + 2 * t;
                  w |= cvt_e2m1x2(__fmul_rn(pv[k + 1], r), __fmul_rn(pv[k], r)) << (8 * t);
                }
                pw[2 * mbk + q] = w;
              }
            }
          }
        }
        if (!__all_sync(FULL, u < 1 || mbar_wait(bar(B_P_FREE), (u - 1) & 1))) { ok = false; break; }
        *reinterpret_cast<uint4*>(smem + SM_P + row * 32 + ((half ^ ((row >> 2) & 1)) * 16)) =
            make_uint4(pw[0], pw[1], pw[2], pw[3]);
        *reinterpret_cast<uint16_t*>(smem + SM_PSF + (row & 31) * 16 + (row >> 5) * 4 + 2 * half) = (uint16_t)sfw;
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_P_FULL));
        if (have_pend && !merge_x4()) { ok = false; break; }
        have_pend = true;
        pend_member = member;
        pend_mb = mb;
        pend_lb = lb;
      }
      if (ok && have_pend) ok = merge_x4();
    }
    if (ok && !__all_sync(FULL, mbar_wait(bar(B_DONE), 0))) ok = false;
    tc_fence_after();
    if (!ok) { raise_timeout(A.status); *abort_flag = 1; }
    // ---- epilogue: O = (2^(m16-m) O + 2^(m8-m) vsc ⊙ o8) / l, vsc the channel
    // scale of whichever low-bit phase ran last (INT8 sv or NVFP4 g)
    {
      // both halves of a row carry partial sums; exchange them
      float* lx = red + 512;  // [2 halves][2 values][128 rows], past the item buffers
      lx[(half * 2 + 0) * 128 + row] = l16;
      lx[(half * 2 + 1) * 128 + row] = l8;
      if (!pair_sync(B_EPI + quarter, 0)) { raise_timeout(A.status); *abort_flag = 1; }
      const float l16t = l16 + lx[((1 - half) * 2 + 0) * 128 + row];
      const float l8t = l8 + lx[((1 - half) * 2 + 1) * 128 + row];
      const float mm = fmaxf(m16, m8);
      const float a16 = m16 == -INFINITY ? 0.f : fast_exp2(m16 - mm);
      const float a8 = m8 == -INFINITY ? 0.f : fast_exp2(m8 - mm);
      const float lt = l16t * a16 + l8t * a8;
      const float il = lt > 0.f ? 1.0f / lt : 0.f;
      uint8_t* ot = smem + SM_Q16 + half * 16384;  // channel half = output sub-tile
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        uint32_t orr[32];
        tmem_ld32(tbase + lane_off + TM_O + half * 64 + c, orr);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int ch = half * 64 + c + 2 * i;
          const float v0 = (a16 * __uint_as_float(orr[2 * i]) + a8 * vsc[ch] * o8[c + 2 * i]) * il;
          const float v1 = (a16 * __uint_as_float(orr[2 * i + 1]) + a8 * vsc[ch + 1] * o8[c + 2 * i + 1]) * il;
          __nv_bfloat162 hb = __floats2bfloat162_rn(v0, v1);
          w[i] = *reinterpret_cast<uint32_t*>(&hb);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = (c >> 3) + q;
          *reinterpret_cast<uint4*>(ot + row * 128 + ((chunk ^ (row & 7)) * 16)) =
              make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
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
__global__ void __launch_bounds__(256) pair_lists_kernel(Geom g, const uint8_t* __restrict__ map,
                                                         uint32_t* __restrict__ plist, int* __restrict__ pcnt,
                                                         int npairs) {
  const int pair = blockIdx.x, bh = blockIdx.y, nb = g.nb;
  const int qa = 2 * pair, qb = (2 * pair + 1 < nb) ? 2 * pair + 1 : -1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint8_t* ra = map + ((size_t)bh * nb + qa) * nb;
  const uint8_t* rb = qb >= 0 ? map + ((size_t)bh * nb + qb) * nb : nullptr;
  uint32_t* out = plist + ((size_t)bh * npairs + pair) * (2 * nb);
  __shared__ int wtot[8];
  int run = 0;
  int counts[3];
  const int phase_bits[3] = {16, 8, 4};
  for (int ph = 0; ph < 3; ++ph) {
    const int start = run;
    for (int base = 0; base < nb; base += 256) {
      const int kb = base + threadIdx.x;
      bool a = false, b = false;
      if (kb < nb) {
        a = ra[kb] == phase_bits[ph];
        b = rb && rb[kb] == phase_bits[ph];
      }
      const unsigned bal = __ballot_sync(0xffffffffu, a || b);
      if (lane == 0) wtot[warp] = __popc(bal);
      __syncthreads();
      if (a || b) {
        int off = run;
        for (int w = 0; w < warp; ++w) off += wtot[w];
        off += __popc(bal & ((1u << lane) - 1u));
        const int rx = kb % g.nrx, ry = (kb / g.nrx) % g.nry;
        const bool full = (ry + 1) * g.rh <= g.Hh && (rx + 1) * g.rw <= g.Ww;
        out[off] = (uint32_t)kb | ((uint32_t)a << 16) | ((uint32_t)b << 17) | ((uint32_t)ph << 18) |
                   ((uint32_t)full << 20);
      }
      for (int w = 0; w < 8; ++w) run += wtot[w];
      __syncthreads();
    }
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

bool attention_tc_supported(const Geom& g) {
  return g.d == kD && encode_fn() != nullptr;
}

cudaError_t launch_pair_lists(const Geom& g, const Layout& L, void* ws, cudaStream_t st) {
  const int npairs = (g.nb + 1) / 2;
  pair_lists_kernel<<<dim3(npairs, g.BH), 256, 0, st>>>(g, at<uint8_t>(ws, L, R_MAP), at<uint32_t>(ws, L, R_PLIST),
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
  e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<<<dim3(A.npairs, g.BH), kThreads, kSmemBytes, st>>>(tq, tk, tv, to, tq8, tk8, tv8, tq4, tk4, tv4,
                                                                      g, A);
  return cudaGetLastError();
}

}  // namespace da2
