// Stage 3 on the Blackwell tensor cores (tcgen05 + TMEM + TMA), head
// dimension 64 or 128, and the own dense bf16 attention on the same kernel.
//
// DraftAttention2 abstract and reading note (Method overview bullets 3-4): one
// kernel runs a phase per precision for each query block, sharing data
// movement, softmax statistics and one output accumulator, and rescaling by the
// quantisation scales at phase boundaries; low-bit precision keeps the
// mid-importance interactions.  DraftAttention (v1) abstract: the output is
// restored to the original token order.
//
// Tile.  A precision is assigned per (query block, key block) pair of 64
// tokens, so one query block gives an M = 64 MMA, which runs the tensor core at
// half rate.  Each CTA owns a pair of neighbouring query blocks (2p, 2p+1) —
// rows 0-63 and 64-127 of one M = 128 tile — and walks the merged key list of
// the pair phase by phase, one key block (a "unit") at a time.  A key block
// only one of the two keeps is computed for all 128 rows and masked for the
// other half.  Nothing a row computes depends on the other query block beyond
// rounding: every quantisation reference below is the row's own per key block,
// and references are powers of two.
//
// Two tiles per CTA.  Tensor-memory kernels run one CTA per SM, so each CTA
// holds two independent tile engines — two query-block pairs, each with its
// own softmax warpgroup, TMA warp, MMA warp, 256 TMEM columns and shared-memory
// half.  While one tile's softmax waits on a TMEM load, a barrier or its MMAs,
// the other's exponentials keep the special-function unit busy, and the
// tensor core alternates between the two tiles' score and P·V MMAs.
//
// Roles (12 warps).  Warps 0-3 (tile 0) and 4-7 (tile 1) do the softmax, one
// thread per tile row (TMEM lane), 64 scores per unit; warps 8 and 10 issue
// the TMA loads of tiles 0 and 1, warps 9 and 11 their MMAs, each from a
// non-blocking scheduler.
//
//   16-bit  S = Q·K^T (kind::f16, fp32 in TMEM, two buffers);
//           P = exp2(s·log2e/√d − m) rounded to bf16 against an integer
//           reference m per row (the shared statistics), raised lazily (O
//           rescaled in TMEM only when the row max grows by more than 2^8); P
//           replaces the scores in TMEM and O += P·V reads it from there (V
//           MN-major from the TMA tile).
//   8-bit   S8 = Q8·K8^T (kind::i8, s32).  Per row and key block the
//           reference is the block's own maximum rounded up to a power of two,
//           2^r_blk: codes c = round(255·2^(x − r_blk)).  c·2^(r_blk − m) is an
//           8-bit integer times a power of two, exact in bf16, and so are the
//           INT8 V codes: O += P·V8 runs on the 16-bit path (kind::f16, P from
//           TMEM) straight into the shared accumulator, every product exact.
//           The row sum takes the same weights /255.
//   4-bit   S = Q4·K4^T (kind::mxf4nvf4, block16 ue4m3 scales copied into
//           TMEM with tcgen05.cp); P = NVFP4 of 2688·2^(x − m) per 16 keys
//           against the shared reference m, raised to the ceiling of the
//           running maximum at the phase start and to a unit's maximum when
//           it exceeds it (which reproduces each block's own power-of-two
//           reference while the microscale stays normal); O += P4·V4 into the
//           shared fp32 accumulator.  The row sum of the quantised weights is
//           exact integer arithmetic in the softmax thread: a byte permute
//           maps four e2m1 codes to twice their values, a 4-way byte dot
//           product adds them, one multiply applies the microscale.
//   Around each low-bit phase O is multiplied by the inverse of the phase's V
//   channel scale (sv/255 or g/2688) and back — the rescaling at the phase
//   boundaries — so that the phase's MMAs work on the codes.
// Operands arrive by TMA: bf16 Q/K/V as 8×8-token region boxes straight from
// the [B,H,N,d] tensors (padding is the TMA zero fill), codes as 2-D boxes of
// the workspace (V's INT8 codes held as bf16 values by the preparation).  Q8
// and Q4 reuse Q's buffer once the last 16-bit score MMA has completed.  The
// epilogue writes O / l through the same region box with a TMA store, whose
// clipping drops the padding rows — the restore.
// Every wait is bounded; on expiry the CTA raises its status word, stops
// issuing, waits (bounded) for its own copies in flight and releases its
// tensor memory.
#include <cuda.h>

#include <climits>
#include <mutex>
#include <type_traits>

#include "da2_internal.cuh"
#include "sm100.cuh"

namespace da2 {
namespace {

using namespace sm100;

constexpr int kTiles = 2;
constexpr int kSoftmaxWarps = 4;  // per tile
constexpr int kIssueWarp0 = 8;    // warps 8 + 2t (TMA) and 9 + 2t (MMA) serve tile t
constexpr int kThreads = 384;  // 168 registers per thread: the SM's 64K registers
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
constexpr uint32_t kDefaultSpin = 1u << 22;

// TMEM columns (512 per CTA, 256 per tile, from the tile's base).  [0, D): O,
// the one fp32 accumulator every phase adds into.  [128, 256): two score buffers of 64 columns (one key block).  The
// 4-bit phase keeps its scores in the second buffer only (its P goes to shared
// memory, so the buffer is free as soon as the softmax has read it) and its
// scale factors over the first: Q 128, K 136/144 (two slots), V 152/156, P
// 160/164 (all 4-aligned, as block-scaled MMAs require).
constexpr uint32_t kTmemCols = 512, kTileCols = 256;
constexpr uint32_t TM_O = 0, TM_S = 128, TM_S4 = 192;
constexpr uint32_t TM_SFQ = 128, TM_SFK = 136, TM_SFV = 152, TM_SFP = 160;

// Shared-memory map: one half per tile (offsets from the tile's base, the
// first 1024-aligned), then the CTA's MISC words.
template <int D>
struct Smem {
  static constexpr int H = D / 64;                         // 64-channel halves of a bf16 row
  static constexpr uint32_t Q = 0;                         // Q16 [H][2 blocks][64 rows][128 B], SW128;
                                                           // later Q8 [128 rows][D B] and Q4 at Q4OFF
  static constexpr uint32_t Q4OFF = 128u * D;              // Q4 [128 rows][D/2 B]
  static constexpr uint32_t KR = 256u * D;                 // K ring
  static constexpr uint32_t STAGE = 128u * D;              // one ring slot: a bf16 key block
  static constexpr uint32_t VR = KR + kStages * STAGE;     // V ring
  static constexpr uint32_t P4 = VR + kStages * STAGE;     // two 4-bit P buffers
  static constexpr uint32_t P4STRIDE = 5120;               // codes [128 rows][32 B] | scale atom
  static constexpr uint32_t P4SF = 4096;
  static constexpr uint32_t VS = P4 + 2 * P4STRIDE;        // fp32 [4][D] channel factors (see VS_*)
  static constexpr uint32_t BAR = VS + ((16u * D + 255u) & ~255u);
  static constexpr uint32_t TILE = (BAR + 256u + 1023u) & ~1023u;
  static constexpr uint32_t MISC = kTiles * TILE;          // TMEM base, abort flag, e4m3 reciprocals
  static constexpr uint32_t BYTES = MISC + 256 + 1024;     // + alignment slack
  // 4-bit slots: K4 (or V4) codes take 32·D bytes; scale atoms follow
  static constexpr uint32_t SL_SF = 32u * D;
};
static_assert(Smem<128>::BYTES <= 227 * 1024, "shared memory");
static_assert(Smem<128>::Q4OFF + 64u * 128 <= Smem<128>::KR, "Q8 and Q4 fit in Q's buffer");

// channel factors that move O into a low-bit phase's units and back:
// 255/sv, sv/255 (INT8: V codes times sv/255... P codes /255), 2688/g, g/2688
// (NVFP4: V/g and 2688 P); 1 where the channel scale is 0
enum { VS_TO8 = 0, VS_FROM8 = 1, VS_TO4 = 2, VS_FROM4 = 3 };

// mbarrier slots (8 bytes each)
enum {
  B_Q16 = 0, B_Q8, B_Q4, B_SFQ, B_QFREE, B_S_FREE, B_K_FULL, B_K_EMPTY = B_K_FULL + kStages,
  B_V_FULL = B_K_EMPTY + kStages, B_V_EMPTY = B_V_FULL + kStages, B_S_FULL = B_V_EMPTY + kStages,
  B_P_FULL = B_S_FULL + 2, B_P_FREE = B_P_FULL + 2, B_DONE = B_P_FREE + 2, B_COUNT
};
static_assert(B_COUNT * 8 <= 256, "barrier area");

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
  uint32_t spin;          // bound of every wait (polls)
  int poison;             // test hook: this CTA skips its first K load (-1: none)
};

__device__ __forceinline__ void raise_timeout(int* status) { atomicOr(status, 1); }

// packed fp32x2 arithmetic (one FMA-pipe instruction for two values)
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
// 2^k for an integer-valued float k <= 127 (exact; 0 below the normal range)
__device__ __forceinline__ float pow2i(float k) { return k > -127.0f ? __int_as_float(((int)k + 127) << 23) : 0.0f; }
// Twice the sum of the eight e2m1 values packed in w (non-negative codes):
// a byte permute looks up 2|v| for four codes at a time (0 1 2 3 4 6 8 12),
// a byte dot product with ones adds them.
__device__ __forceinline__ int e2m1_sum2(uint32_t w, int acc) {
  constexpr uint32_t kLo = 0x03020100u, kHi = 0x0C080604u;
  acc = __dp4a(__byte_perm(kLo, kHi, w & 0xffffu), 0x01010101u, (unsigned)acc);
  return (int)__dp4a(__byte_perm(kLo, kHi, w >> 16), 0x01010101u, (unsigned)acc);
}
// value of a ue4m3 scale: 2^(e-7) (1 + m/8), or m 2^-9 when e = 0
__device__ __forceinline__ float ue4m3_value(uint32_t sf) {
  const uint32_t ex = sf >> 3, mt = sf & 7u;
  return ex ? __uint_as_float(((ex + 120u) << 23) | (mt << 20)) : (float)mt * (1.0f / 512.0f);
}

// Items: kb | inA << 16 | inB << 17 | kind << 18 | full << 20 (the key block
// has no padding slot).
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

// kDense: every key block in the 16-bit phase, items generated in the kernel
// (a separate instantiation, so that the sparse kernel carries none of it)
template <int D, bool kDense>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const __grid_constant__ CUtensorMap tmQ8, const __grid_constant__ CUtensorMap tmK8,
               const __grid_constant__ CUtensorMap tmV8, const __grid_constant__ CUtensorMap tmQ4,
               const __grid_constant__ CUtensorMap tmK4, const __grid_constant__ CUtensorMap tmV4, Geom g,
               TcArgs A) {
  using SM = Smem<D>;
  constexpr int H = SM::H;
  // a CTA that timed out raised the status word: later CTAs skip their work
  if (*reinterpret_cast<volatile const int*>(A.status) != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s0 = (uint32_t)__cvta_generic_to_shared(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this warp's tile: its query-block pair, shared-memory half and TMEM columns
  const int t = warp < kIssueWarp0 ? warp / kSoftmaxWarps : (warp - kIssueWarp0) >> 1;
  const long long gi = (long long)kTiles * blockIdx.x + t;
  const bool active = gi < (long long)A.npairs * g.BH;
  const int bh = active ? (int)(gi / A.npairs) : 0, pair = active ? (int)(gi - (long long)bh * A.npairs) : 0;
  uint8_t* ts = smem + t * SM::TILE;
  const uint32_t s0t = s0 + t * SM::TILE;
  const int qa = 2 * pair, qb = (2 * pair + 1 < g.nb) ? 2 * pair + 1 : -1;
  const size_t prow = (size_t)bh * A.npairs + pair;
  const int4 pc = !active ? make_int4(0, 0, 0, 0)
                 : kDense ? make_int4(g.nb, 0, 0, 0) : *reinterpret_cast<const int4*>(A.pcnt + prow * 4);
  // one key block per unit: units [0, nu16) 16-bit, [nu16, nu8) INT8, [nu8, nu) 4-bit
  const int nu16 = pc.x, nu8 = pc.x + pc.y, nu = pc.x + pc.y + pc.z;
  const uint32_t* items = kDense ? nullptr : A.plist + prow * (size_t)(2 * g.nb);
  const uint32_t spin = A.spin;
  // entry i of the pair's list; in dense mode key block i, kept by both query
  // blocks, flagged full unless it holds the ragged tail
  auto item_at = [&](int i) -> uint32_t {
    if (!kDense) return items[i];
    return (uint32_t)i | (1u << 16) | ((2 * pair + 1 < g.nb ? 1u : 0u) << 17) |
           ((uint32_t)((i + 1) * 64 <= g.N) << 20);
  };
  auto bar = [&](int i) { return s0t + SM::BAR + 8u * (uint32_t)i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + SM::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::MISC + 8);
  // 1 / (1 + m/8) for m = 0..7, then 1 / m (0 for m = 0): reciprocals of e4m3 scales
  float* rcp_tab = reinterpret_cast<float*>(smem + SM::MISC + 64);
  float* vsc = reinterpret_cast<float*>(ts + SM::VS);  // [4][D] channel factors (VS_*)
  if (threadIdx.x < 16)
    rcp_tab[threadIdx.x] = threadIdx.x < 8 ? 8.0f / (float)(8 + threadIdx.x)
                                           : (threadIdx.x > 8 ? 1.0f / (float)(threadIdx.x - 8) : 0.f);

  if (threadIdx.x == 0) {
    for (int tt = 0; tt < kTiles; ++tt) {
      auto tbar = [&](int i) { return s0 + tt * SM::TILE + SM::BAR + 8u * (uint32_t)i; };
      mbar_init(tbar(B_Q16), 1);
      mbar_init(tbar(B_Q8), 1);
      mbar_init(tbar(B_Q4), 1);
      mbar_init(tbar(B_SFQ), kSoftmaxWarps);     // each softmax warp wrote Q's scale factors in its lanes
      mbar_init(tbar(B_QFREE), 1);               // the last 16-bit score MMA (the last reader of Q16) completed
      mbar_init(tbar(B_S_FREE), kSoftmaxWarps);  // per 4-bit unit: its scores were read
      for (int s = 0; s < kStages; ++s) {
        mbar_init(tbar(B_K_FULL + s), 1); mbar_init(tbar(B_K_EMPTY + s), 1);
        mbar_init(tbar(B_V_FULL + s), 1); mbar_init(tbar(B_V_EMPTY + s), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(tbar(B_S_FULL + b), 1);
        mbar_init(tbar(B_P_FULL + b), kSoftmaxWarps);  // per unit parity: P of unit u written
        mbar_init(tbar(B_P_FREE + b), 1);              // the P·V of unit u has completed
      }
      mbar_init(tbar(B_DONE), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kIssueWarp0 + 1) tmem_alloc(s0 + SM::MISC, kTmemCols);
  if (!kDense && warp < kIssueWarp0) {
    // each softmax warpgroup fills its own tile's channel factors
    for (int c = threadIdx.x & 127; c < D; c += 128) {
      const float sv = nu8 > nu16 ? A.v_s8[(size_t)bh * D + c] : 0.f, gv = nu > nu8 ? A.v_g4[(size_t)bh * D + c] : 0.f;
      vsc[VS_TO8 * D + c] = sv > 0.f ? 255.0f / sv : 1.0f;
      vsc[VS_FROM8 * D + c] = sv > 0.f ? sv / 255.0f : 1.0f;
      vsc[VS_TO4 * D + c] = gv > 0.f ? kP4Range / gv : 1.0f;
      vsc[VS_FROM4 * D + c] = gv > 0.f ? gv / kP4Range : 1.0f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];
  const uint32_t tcol = tbase + (uint32_t)t * kTileCols;  // this tile's TMEM columns

  const int t_of = g.nry * g.nrx;  // blocks per frame
  auto box = [&](int blk, int& cx, int& cy, int& cf) {
    const int tf = blk / t_of, rem = blk - tf * t_of;
    const int ry = rem / g.nrx, rx = rem - ry * g.nrx;
    cx = rx * g.rw; cy = ry * g.rh; cf = bh * g.T + tf;
  };

  if (warp >= kIssueWarp0) {
  // the third warpgroup: each tile's TMA producer and MMA issuer
  if (((warp - kIssueWarp0) & 1) == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (elect_one()) {
      prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmV);
      int cx, cy, cf;
      const bool q16 = nu16 > 0, q8 = nu8 > nu16, q4 = nu > nu8;
      if (q16) {
        mbar_expect_tx(bar(B_Q16), (qb >= 0 ? 2u : 1u) * 128u * D);
        box(qa, cx, cy, cf);
        for (int h = 0; h < H; ++h) tma_load_4d(s0t + SM::Q + h * 16384, &tmQ, bar(B_Q16), 64 * h, cx, cy, cf);
        if (qb >= 0) {
          box(qb, cx, cy, cf);
          for (int h = 0; h < H; ++h)
            tma_load_4d(s0t + SM::Q + h * 16384 + 8192, &tmQ, bar(B_Q16), 64 * h, cx, cy, cf);
        }
      }
      // Q8 and Q4 go into Q16's buffer once its last reader has completed
      bool qlow = !(q8 || q4);
      // K of a unit is needed first (scores) and released first; V waits for
      // the P·V two units back.  Issue whichever ring has room, K first.
      int kn = 0, vn = 0;
      int last_k[kStages] = {-1, -1}, last_v[kStages] = {-1, -1};  // last unit loaded into each slot
      uint32_t idle = 0;
      while (kn < nu || vn < nu || !qlow) {
        bool progressed = false;
        if (!qlow && (!q16 || mbar_test(bar(B_QFREE), 0))) {
          if (q8) {
            mbar_expect_tx(bar(B_Q8), (qb >= 0 ? 2u : 1u) * 64u * D);
            tma_load_2d(s0t + SM::Q, &tmQ8, bar(B_Q8), 0, (bh * g.nb + qa) * 64);
            if (qb >= 0) tma_load_2d(s0t + SM::Q + 64 * D, &tmQ8, bar(B_Q8), 0, (bh * g.nb + qb) * 64);
          }
          if (q4) {
            mbar_expect_tx(bar(B_Q4), (qb >= 0 ? 2u : 1u) * 32u * D);
            tma_load_2d(s0t + SM::Q + SM::Q4OFF, &tmQ4, bar(B_Q4), 0, (bh * g.nb + qa) * 64);
            if (qb >= 0) tma_load_2d(s0t + SM::Q + SM::Q4OFF + 32 * D, &tmQ4, bar(B_Q4), 0, (bh * g.nb + qb) * 64);
          }
          qlow = true;
          progressed = true;
        }
        if (kn < nu && (kn < kStages || mbar_test(bar(B_K_EMPTY + kn % kStages), ((kn / kStages) - 1) & 1))) {
          const int kb = item_kb(item_at(kn));
          const uint32_t dst = s0t + SM::KR + (kn % kStages) * SM::STAGE;
          const uint32_t fb = bar(B_K_FULL + kn % kStages);
          if (kn == 0 && (int)blockIdx.x == A.poison) {
            // test hook: this load is never issued, so its consumers' bounded waits expire
          } else if (kn < nu16) {
            mbar_expect_tx(fb, 128u * D);
            box(kb, cx, cy, cf);
            for (int h = 0; h < H; ++h) tma_load_4d(dst + h * 8192, &tmK, fb, 64 * h, cx, cy, cf);
            last_k[kn % kStages] = kn;
          } else if (kn < nu8) {
            mbar_expect_tx(fb, 64u * D);
            tma_load_2d(dst, &tmK8, fb, 0, (bh * g.nb + kb) * 64);
            last_k[kn % kStages] = kn;
          } else {
            const size_t kl = (size_t)bh * g.nb + kb;
            mbar_expect_tx(fb, 32u * D + H * kSfAtomBytes);
            tma_load_2d(dst, &tmK4, fb, 0, (int)(kl * 64));
            bulk_load(dst + SM::SL_SF, A.k_sf4 + kl * H * kSfAtomBytes, H * kSfAtomBytes, fb);
            last_k[kn % kStages] = kn;
          }
          ++kn;
          progressed = true;
        }
        if (vn < kn && (vn < kStages || mbar_test(bar(B_V_EMPTY + vn % kStages), ((vn / kStages) - 1) & 1))) {
          const int kb = item_kb(item_at(vn));
          const uint32_t dst = s0t + SM::VR + (vn % kStages) * SM::STAGE;
          const uint32_t fb = bar(B_V_FULL + vn % kStages);
          if (vn < nu16) {
            mbar_expect_tx(fb, 128u * D);
            box(kb, cx, cy, cf);
            for (int h = 0; h < H; ++h) tma_load_4d(dst + h * 8192, &tmV, fb, 64 * h, cx, cy, cf);
          } else if (vn < nu8) {
            // the INT8 codes as bf16 values, [64 slots][D] per block: the 16-bit tile layout
            mbar_expect_tx(fb, 128u * D);
            for (int h = 0; h < H; ++h) tma_load_2d(dst + h * 8192, &tmV8, fb, 64 * h, (bh * g.nb + kb) * 64);
          } else {
            const size_t kl = (size_t)bh * g.nb + kb;
            mbar_expect_tx(fb, 32u * D + kSfAtomBytes);
            tma_load_2d(dst, &tmV4, fb, 0, (int)(kl * D));
            bulk_load(dst + SM::SL_SF, A.v_sf4 + kl * kSfAtomBytes, kSfAtomBytes, fb);
          }
          last_v[vn % kStages] = vn;
          ++vn;
          progressed = true;
        }
        if (progressed) {
          idle = 0;
        } else if (++idle > spin || *abort_flag) {
          raise_timeout(A.status); *abort_flag = 1;
          break;
        } else {
          __nanosleep(64);  // leave the issue slots of this sub-partition to the softmax warps
        }
      }
      // every copy this CTA issued lands before the CTA may leave (bounded)
      if (q16) (void)mbar_wait(bar(B_Q16), 0, spin);
      if (qlow && q8) (void)mbar_wait(bar(B_Q8), 0, spin);
      if (qlow && q4) (void)mbar_wait(bar(B_Q4), 0, spin);
      for (int s = 0; s < kStages; ++s) {
        if (last_k[s] >= 0) (void)mbar_wait(bar(B_K_FULL + s), (uint32_t)(last_k[s] / kStages) & 1u, spin);
        if (last_v[s] >= 0) (void)mbar_wait(bar(B_V_FULL + s), (uint32_t)(last_v[s] / kStages) & 1u, spin);
      }
    }
  } else {
    // ---------------------------------------------------------------- MMA scheduler
    if (elect_one()) {
      const uint32_t id16 = idesc(kDF32, kFmtBF16, kFmtBF16, false, false, 128, 64);
      const uint32_t idpv = idesc(kDF32, kFmtBF16, kFmtBF16, false, true, 128, D);
      const uint32_t id8 = idesc(kDS32, kFmtS8, kFmtS8, false, false, 128, 64);
      const uint32_t id4s = idesc_f4(128, 64), id4pv = idesc_f4(128, D);
      constexpr uint32_t kSbo8 = 8u * D;                       // INT8 rows of D bytes
      constexpr Swizzle kSw8 = D == 128 ? SW_128 : SW_64;
      constexpr uint32_t kSbo4 = 4u * D;                       // NVFP4 rows of D/2 bytes
      constexpr Swizzle kSw4 = D == 128 ? SW_64 : SW_32;
      bool q16_ready = nu16 == 0, q8_ready = nu8 == nu16, f4_ready = nu == nu8;
      bool ok = true;
      int sn = 0, pn = 0;  // next unit for S, next unit for P·V
      uint32_t idle = 0;
      // the P·V of unit j (and every MMA before it) has completed
      auto pv_done = [&](int j) { return j < 0 || mbar_test(bar(B_P_FREE + (j & 1)), (uint32_t)(j >> 1) & 1u); };
      while (ok && pn < nu) {
        bool progressed = false;
        if (sn < nu) {
          const int s = sn % kStages, b = sn & 1;
          bool can;
          if (sn < nu16) {
            if (!q16_ready) q16_ready = mbar_test(bar(B_Q16), 0);
            // a score buffer is free once the P·V of the unit two back (whose P sat in it) completed
            can = q16_ready && pv_done(sn - 2);
          } else if (sn < nu8) {
            if (!q8_ready) q8_ready = mbar_test(bar(B_Q8), 0);
            can = q8_ready && pv_done(sn - 2);
          } else {
            // Q4 landed and the softmax wrote Q's scale factors, after every
            // earlier P·V completed; afterwards the single 4-bit score buffer
            // is free once the softmax has read the previous unit's scores
            if (!f4_ready) f4_ready = mbar_test(bar(B_Q4), 0) && mbar_test(bar(B_SFQ), 0);
            can = f4_ready && (sn == nu8 || mbar_test(bar(B_S_FREE), (uint32_t)(sn - 1 - nu8) & 1u));
          }
          if (can && mbar_test(bar(B_K_FULL + s), (sn / kStages) & 1)) {
            tc_fence_after();
            const uint32_t st = s0t + SM::KR + s * SM::STAGE;
            if (sn < nu16) {
              const uint32_t sd = tcol + TM_S + 64u * b;
#pragma unroll
              for (int k = 0; k < D / 16; ++k) {
                const int h = k >> 2, kk = k & 3;
                mma_f16(sd, smem_desc(s0t + SM::Q + h * 16384 + kk * 32, 16, 1024, SW_128),
                        smem_desc(st + h * 8192 + kk * 32, 16, 1024, SW_128), id16, k > 0 ? 1u : 0u);
              }
            } else if (sn < nu8) {
              const uint32_t sd = tcol + TM_S + 64u * b;
#pragma unroll
              for (int kk = 0; kk < D / 32; ++kk)
                mma_i8(sd, smem_desc(s0t + SM::Q + kk * 32, 16, kSbo8, kSw8), smem_desc(st + kk * 32, 16, kSbo8, kSw8),
                       id8, kk > 0 ? 1u : 0u);
            } else {
              const uint32_t sfk = tcol + TM_SFK + 8u * b;
#pragma unroll
              for (int c = 0; c < H; ++c) {
                tc_cp_atom(sfk + 4 * c, st + SM::SL_SF + c * kSfAtomBytes);
                mma_f4(tcol + TM_S4, smem_desc(s0t + SM::Q + SM::Q4OFF + 32 * c, 16, kSbo4, kSw4),
                       smem_desc(st + 32 * c, 16, kSbo4, kSw4), id4s, c > 0 ? 1u : 0u, tcol + TM_SFQ + 4 * c,
                       sfk + 4 * c);
              }
            }
            mma_commit(bar(B_S_FULL + b));
            mma_commit(bar(B_K_EMPTY + s));
            if (sn == nu16 - 1) mma_commit(bar(B_QFREE));
            ++sn;
            progressed = true;
          }
        }
        if (pn < sn) {
          const int s = pn % kStages;
          if (mbar_test(bar(B_V_FULL + s), (pn / kStages) & 1) && mbar_test(bar(B_P_FULL + (pn & 1)), (pn >> 1) & 1)) {
            tc_fence_after();
            const uint32_t st = s0t + SM::VR + s * SM::STAGE;
            if (pn < nu8) {
              // 16-bit and INT8 units: P (bf16) from TMEM, V tiles MN-major bf16
              const uint32_t pt = tcol + TM_S + 64u * (pn & 1);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_f16_ta(tcol + TM_O, pt + 8 * kk, smem_desc(st + kk * 2048, 8192, 1024, SW_128), idpv, 1u);
            } else {
              const uint32_t pb = s0t + SM::P4 + (pn & 1) * SM::P4STRIDE;
              const uint32_t sfv = tcol + TM_SFV + 4u * (pn & 1), sfp = tcol + TM_SFP + 4u * (pn & 1);
              tc_cp_atom(sfv, st + SM::SL_SF);
              tc_cp_atom(sfp, pb + SM::P4SF);
              mma_f4(tcol + TM_O, smem_desc(pb, 16, 256, SW_32), smem_desc(st, 16, 256, SW_32), id4pv, 1u, sfp, sfv);
            }
            mma_commit(bar(B_P_FREE + (pn & 1)));
            mma_commit(bar(B_V_EMPTY + s));
            ++pn;
            progressed = true;
          }
        }
        if (progressed) {
          idle = 0;
        } else if (++idle > spin || *abort_flag) {
          ok = false;
        } else {
          __nanosleep(32);  // leave the issue slots of this sub-partition to the softmax warps
        }
      }
      mma_commit(bar(B_DONE));
      if (!ok) { raise_timeout(A.status); *abort_flag = 1; }
    }
  }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-7
    const int row = threadIdx.x & 127;               // TMEM lane and tile row
    const int wq = warp & 3;                         // lane quarter
    const bool in_b = row >= 64;
    const int qrow_blk = in_b ? qb : qa;
    const uint32_t tl = tcol + ((uint32_t)(wq * 32) << 16);  // this warp's lane quarter
    const float sl2 = kLog2e * rsqrtf((float)D);
    const float sq = (!kDense && nu8 > nu16 && qrow_blk >= 0) ? A.q_s8[(size_t)bh * g.nb + qrow_blk] : 0.f;
    const unsigned FULL = 0xffffffffu;
    // the P·V of unit v (and every MMA before it) has completed
    auto pfree_wait = [&](int v) -> bool {
      return v < 0 || mbar_wait(bar(B_P_FREE + (v & 1)), (uint32_t)(v >> 1) & 1u, spin);
    };
    float ref = -INFINITY;    // O's reference per row: an integer, log2 units (the shared statistics)
    float l = 0.f;            // the row sum, relative to 2^ref
    float x_run = -INFINITY;  // running row max (log2 units) over every unit so far
    bool ok = true;
#pragma unroll
    for (int c = 0; c < D; c += 32) tmem_fill32(tl + TM_O + c, 0u);  // O starts at zero
    tmem_wait_st();
    // item entries (and INT8 key scales) are loaded one unit ahead, so no unit
    // starts by waiting on global memory
    auto item_for = [&](int v) -> uint32_t { return v < nu ? item_at(v) : 0u; };
    auto sk_for = [&](int v, uint32_t ev) -> float {
      return (v >= nu16 && v < nu8) ? A.k_s8[(size_t)bh * g.nb + item_kb(ev)] : 0.f;
    };
    uint32_t e_next = item_for(0);
    float sk_next = sk_for(0, e_next);
    auto member_of = [&](uint32_t e) -> bool { return ((e >> (in_b ? 17 : 16)) & 1u) != 0; };
    // O (this thread's row) times a per-row factor a and per-channel factors
    // ch[] (ch == nullptr: none); the MMAs that write O have completed
    auto scale_o = [&](float a, const float* ch) {
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t orr[32];
        tmem_ld32(tl + TM_O + c, orr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          orr[i] = __float_as_uint(__uint_as_float(orr[i]) * (ch ? a * ch[c + i] : a));
        tmem_st32(tl + TM_O + c, orr);
      }
      tmem_wait_st();
    };
    // the lazy reference of the 16-bit and INT8 phases: raised to ceil(um)
    // only when the unit's row maximum um exceeds it by more than 2^8; returns
    // the factor that O and l take (1 if unchanged)
    auto lazy_raise = [&](float um, bool& need_o) -> float {
      const bool need = um != -INFINITY && (ref == -INFINITY || um > ref + kRescaleThreshold);
      need_o = need && ref != -INFINITY;
      const float a = need_o ? pow2i(ref - ceilf(um)) : 1.0f;
      if (need) ref = ceilf(um);
      return a;
    };
    // a unit's P goes to TMEM in place of its scores; O, if its reference
    // moved, is rescaled first (once the P·V of the unit before completed)
    auto finish_unit = [&](int u, uint32_t sb, const uint32_t* pw, bool need_o, float a) -> bool {
      if (__any_sync(FULL, need_o)) {
        if (!__all_sync(FULL, pfree_wait(u - 1))) return false;
        tc_fence_after();
        scale_o(a, nullptr);
      }
      tmem_st32(sb, pw);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P_FULL + (u & 1)));
      return true;
    };
    // the last P·V before a phase boundary has completed (and O may be read)
    auto boundary = [&](int last) -> bool {
      if (last < 0) return true;
      const bool done = __all_sync(FULL, pfree_wait(last));
      tc_fence_after();
      return done;
    };

    // ================================================================ 16-bit phase
    for (int u = 0; ok && u < nu16; ++u) {
      if ((u & 7) == 0 && __any_sync(FULL, *abort_flag != 0)) { ok = false; break; }
      const uint32_t sb = tl + TM_S + 64u * (u & 1);
      if (!__all_sync(FULL, mbar_wait(bar(B_S_FULL + (u & 1)), (u >> 1) & 1, spin))) { ok = false; break; }
      tc_fence_after();
      const uint32_t e = e_next;
      const bool member = member_of(e);
      e_next = item_for(u + 1);
      uint32_t sr[64];
      tmem_ld32(sb, sr);
      tmem_ld32(sb + 32, sr + 32);
      tmem_wait_ld();
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
      sk_next = sk_for(u + 1, e_next);
      const float um = mx * sl2;  // the unit's row max, log2 units
      x_run = fmaxf(x_run, um);
      bool need_o;
      const float a = lazy_raise(um, need_o);
      uint32_t pw[32];
      if (member) {
        const uint64_t sl2x2 = f2pack(sl2, sl2), negm = f2pack(-ref, -ref);
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
        float s0_, s1_, s2_, s3_;
        f2unpack(f2add(acc[0], acc[1]), s0_, s1_);
        f2unpack(f2add(acc[2], acc[3]), s2_, s3_);
        l = l * a + ((s0_ + s1_) + (s2_ + s3_));
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pw[i] = 0u;
        l *= a;
      }
      if (!finish_unit(u, sb, pw, need_o, a)) { ok = false; break; }
    }

    // ================================================================ INT8 phase
    if (ok && nu8 > nu16) {
      // O goes to INT8 units (divided by the V channel scale sv/255)
      ok = boundary(nu16 - 1);
      if (ok) scale_o(1.0f, vsc + VS_TO8 * D);
      for (int u = nu16; ok && u < nu8; ++u) {
        if ((u & 7) == 0 && __any_sync(FULL, *abort_flag != 0)) { ok = false; break; }
        const uint32_t sb = tl + TM_S + 64u * (u & 1);
        if (!__all_sync(FULL, mbar_wait(bar(B_S_FULL + (u & 1)), (u >> 1) & 1, spin))) { ok = false; break; }
        tc_fence_after();
        const uint32_t e = e_next;
        const float sk = sk_next;
        const bool member = member_of(e);
        e_next = item_for(u + 1);
        uint32_t sr[64];
        tmem_ld32(sb, sr);
        tmem_ld32(sb + 32, sr + 32);
        tmem_wait_ld();
        const unsigned long long vm = item_full(e) ? ~0ull : key_mask(g, item_kb(e));
        const bool full = vm == ~0ull;
        const float sc = sq * sk * sl2;  // score scale, log2 units (>= 0)
        float xh = -INFINITY;
        if (member) {
          // the row max on the integer scores (padding keys at INT_MIN)
          if (!full) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (!((vm >> i) & 1ull)) sr[i] = 0x80000000u;
          }
          int m4[4] = {INT_MIN, INT_MIN, INT_MIN, INT_MIN};
#pragma unroll
          for (int i = 0; i < 64; i += 8)
#pragma unroll
            for (int q = 0; q < 4; ++q) m4[q] = max(m4[q], max((int)sr[i + 2 * q], (int)sr[i + 2 * q + 1]));
          xh = (float)max(max(m4[0], m4[1]), max(m4[2], m4[3])) * sc;  // a member row has a real key
        }
        sk_next = sk_for(u + 1, e_next);
        const float um = xh;
        x_run = fmaxf(x_run, um);
        bool need_o;
        const float a = lazy_raise(um, need_o);
        uint32_t pw[32];
        if (member) {
          // codes c = round(255 p), p = 2^(s*sc - rb) against the block's own
          // power-of-two reference rb; P = c * 2^(rb - ref), exact in bf16
          const float rb = ceilf(xh);
          const float s2k = pow2i(rb - ref);  // rb - ref <= 8
          const uint64_t scx2 = f2pack(sc, sc), negr = f2pack(-rb, -rb), kx2 = f2pack(-kI8BiasF, -kI8BiasF);
          const uint64_t c255 = f2pack(255.0f, 255.0f), kmag = f2pack(kI8BiasF, kI8BiasF);
          const uint64_t k2 = f2pack(s2k, s2k), nmk = f2pack(-kI8BiasF * s2k, -kI8BiasF * s2k);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int k0 = 2 * i;
            // the exact s32 -> fp32 conversion through the mantissa of 1.5*2^23 (|S| < 2^22)
            const uint64_t sp = f2add(f2pack(__uint_as_float(sr[k0] + kI8Bias), __uint_as_float(sr[k0 + 1] + kI8Bias)), kx2);
            float x0, x1;
            f2unpack(f2fma(sp, scx2, negr), x0, x1);
            float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            if (!full) {  // padding keys contribute nothing, whatever the block scale (sc may be 0)
              if (!((vm >> k0) & 1ull)) p0 = 0.f;
              if (!((vm >> (k0 + 1)) & 1ull)) p1 = 0.f;
            }
            // 255 p + 1.5*2^23 holds the round-to-nearest-even code; times 2^k minus 1.5*2^23*2^k is c*2^k exactly
            const uint64_t w2 = f2fma(f2fma(f2pack(p0, p1), c255, kmag), k2, nmk);
            acc[i & 3] = f2add(acc[i & 3], w2);
            float w0, w1;
            f2unpack(w2, w0, w1);
            pw[i] = __byte_perm(__float_as_uint(w0), __float_as_uint(w1), 0x7632);  // the two bf16 halves
          }
          float s0_, s1_, s2_, s3_;
          f2unpack(f2add(acc[0], acc[1]), s0_, s1_);
          f2unpack(f2add(acc[2], acc[3]), s2_, s3_);
          l = l * a + ((s0_ + s1_) + (s2_ + s3_)) * (1.0f / 255.0f);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) pw[i] = 0u;
          l *= a;
        }
        if (!finish_unit(u, sb, pw, need_o, a)) { ok = false; break; }
      }
      // back to value units
      if (ok) ok = boundary(nu8 - 1);
      if (ok) scale_o(1.0f, vsc + VS_FROM8 * D);
    }

    // ================================================================ 4-bit phase
    if (ok && nu > nu8) {
      // O goes to 4-bit units (divided by g/2688), against a reference raised
      // to the ceiling of the running maximum, so that the phase's P stays in
      // (0, 1] and later raises are rare
      ok = boundary(nu8 - 1);
      const float r0 = x_run == -INFINITY ? ref : (ref == -INFINITY ? ceilf(x_run) : fmaxf(ref, ceilf(x_run)));
      const float a0 = (ref == -INFINITY || r0 == ref) ? 1.0f : pow2i(ref - r0);
      ref = r0;
      l *= a0;
      if (ok) {
        scale_o(a0, vsc + VS_TO4 * D);
        // Q's scale factors into TMEM (the columns of the first score buffer,
        // free now that every earlier P·V has completed): this warp writes its
        // lane quarter, lane i the scales of rows i, i+32 (query block a) and
        // i+64, i+96 (query block b) per 64-channel chunk
        const uint32_t tq = tl;
#pragma unroll
        for (int c = 0; c < H; ++c) {
          uint32_t w[4];
          const uint8_t* sa = A.q_sf4 + ((size_t)bh * g.nb + qa) * H * kSfAtomBytes + c * kSfAtomBytes + lane * 16;
          w[0] = *reinterpret_cast<const uint32_t*>(sa);
          w[1] = *reinterpret_cast<const uint32_t*>(sa + 4);
          if (qb >= 0) {
            const uint8_t* sbp = A.q_sf4 + ((size_t)bh * g.nb + qb) * H * kSfAtomBytes + c * kSfAtomBytes + lane * 16;
            w[2] = *reinterpret_cast<const uint32_t*>(sbp);
            w[3] = *reinterpret_cast<const uint32_t*>(sbp + 4);
          } else {
            w[2] = w[3] = 0u;
          }
          tmem_st4(tq + TM_SFQ + 4 * c, w);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_SFQ));
      }
      for (int u = nu8; ok && u < nu; ++u) {
        if ((u & 7) == 0 && __any_sync(FULL, *abort_flag != 0)) { ok = false; break; }
        const uint32_t sb = tl + TM_S4;
        if (!__all_sync(FULL, mbar_wait(bar(B_S_FULL + (u & 1)), (u >> 1) & 1, spin))) { ok = false; break; }
        tc_fence_after();
        const uint32_t e = e_next;
        const bool member = member_of(e);
        e_next = item_for(u + 1);
        uint32_t sr[64];
        tmem_ld32(sb, sr);
        tmem_ld32(sb + 32, sr + 32);
        tmem_wait_ld();
        // the scores are in registers: the MMA warp may overwrite the buffer
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_FREE));
        const unsigned long long vm = item_full(e) ? ~0ull : key_mask(g, item_kb(e));
        float mx = -INFINITY;
        if (member) {
          if (vm != ~0ull) {
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
          mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * sl2;
        }
        const float um = mx;  // the unit's row maximum
        // the reference rises to ceil(max) whenever the max exceeds it: O is
        // rescaled first, once the P·V of the unit before completed
        const bool raise = um != -INFINITY && (ref == -INFINITY || um > ref);
        const float a = (raise && ref != -INFINITY) ? pow2i(ref - ceilf(um)) : 1.0f;
        if (__any_sync(FULL, raise)) {
          if (!__all_sync(FULL, pfree_wait(u - 1))) { ok = false; break; }
          tc_fence_after();
          scale_o(a, nullptr);
        }
        if (raise) { l *= a; ref = ceilf(um); }
        uint32_t pw[8];
        uint32_t sfw = 0u;  // the row's four e4m3 P scales
#pragma unroll
        for (int i = 0; i < 8; ++i) pw[i] = 0u;
        if (member) {
          const uint64_t sl2x2 = f2pack(sl2, sl2), negr = f2pack(-ref, -ref);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float x0, x1;
            f2unpack(f2fma(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), sl2x2, negr), x0, x1);
            sr[2 * i] = __float_as_uint(fast_exp2(x0));
            sr[2 * i + 1] = __float_as_uint(fast_exp2(x1));
          }
          // NVFP4 of 2688 p over 16 consecutive keys: e4m3 scale from the microblock max / 6
          float lq = 0.f;  // sum of the quantised weights, in units of 2688 / 2
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
            int s2 = 0;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              uint32_t w = 0;
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const int k = 16 * mbk + 8 * q + 2 * t;
                w |= cvt_e2m1x2(__uint_as_float(sr[k + 1]) * rr, __uint_as_float(sr[k]) * rr) << (8 * t);
              }
              pw[2 * mbk + q] = w;
              s2 = e2m1_sum2(w, s2);
            }
            lq = fmaf(ue4m3_value(sf), (float)s2, lq);
          }
          l = fmaf(lq, 0.5f / kP4Range, l);
        }
        // P4 goes to shared memory buffer u&1, free once the P·V of unit u-2 completed
        if (u - 2 >= nu8 && !__all_sync(FULL, pfree_wait(u - 2))) { ok = false; break; }
        uint8_t* pb = ts + SM::P4 + (u & 1) * SM::P4STRIDE;
#pragma unroll
        for (int c = 0; c < 2; ++c)
          *reinterpret_cast<uint4*>(pb + row * 32 + ((c ^ ((row >> 2) & 1)) * 16)) =
              make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
        *reinterpret_cast<uint32_t*>(pb + SM::P4SF + (row & 31) * 16 + (row >> 5) * 4) = sfw;
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_P_FULL + (u & 1)));
      }
      // O returns to value units
      if (ok) ok = boundary(nu - 1);
      if (ok) scale_o(1.0f, vsc + VS_FROM4 * D);
    }
    if (!ok) { raise_timeout(A.status); *abort_flag = 1; }
    // ---- epilogue: O / l in bf16, staged for the TMA store
    {
      if (ok && nu16 == nu && nu > 0) {
        // only the 16-bit phase ran: its last P·V completes before O is read
        if (!boundary(nu - 1)) { raise_timeout(A.status); *abort_flag = 1; }
      }
      const float il = l > 0.f ? 1.0f / l : 0.f;
      const int r = row & 63;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t orr[32];
        tmem_ld32(tl + TM_O + c, orr);
        tmem_wait_ld();
        uint8_t* ot = ts + SM::Q + (c >> 6) * 16384 + (in_b ? 8192 : 0) + r * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(orr[8 * q + 2 * i]) * il,
                                                      __uint_as_float(orr[8 * q + 2 * i + 1]) * il);
            w[i] = *reinterpret_cast<uint32_t*>(&hb);
          }
          const int chunk = ((c & 63) >> 3) + q;  // 16-byte chunk inside the 128-byte row
          *reinterpret_cast<uint4*>(ot + ((chunk ^ (r & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_async_smem();
    }
  }
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x & 127) == 0 && warp < kIssueWarp0 && active && !*abort_flag) {
    // the first thread of each softmax warpgroup stores its tile
    int cx, cy, cf;
    for (int blk = 0; blk < 2; ++blk) {
      const int qq = blk ? qb : qa;
      if (qq < 0) break;
      box(qq, cx, cy, cf);
      for (int h = 0; h < H; ++h)
        asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                     ::"l"(&tmO), "r"(s0t + SM::Q + h * 16384 + blk * 8192), "r"(64 * h), "r"(cx), "r"(cy), "r"(cf)
                     : "memory");
    }
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
  __syncthreads();
  tc_fence_after();
  if (warp == kIssueWarp0 + 1) {
    // every issued MMA of both tiles has completed before the columns are released
    bool done = true;
    for (int tt = 0; tt < kTiles; ++tt)
      done = mbar_wait(s0 + tt * SM::TILE + SM::BAR + 8u * B_DONE, 0, spin) && done;
    (void)__all_sync(0xffffffffu, done);
    tmem_relinquish();
    tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace
}  // namespace da2

// ------------------------------------------------------------------ host side
namespace da2 {
namespace {

// Merged key lists of query-block pairs (2p, 2p+1): per phase (16, 8, 4) the
// key blocks either member keeps in that phase, ascending, with member flags
// and a flag for key blocks without padding.  The two map rows are staged in
// shared memory once for all passes.
__global__ void __launch_bounds__(256) pair_lists_kernel(Geom g, const uint8_t* __restrict__ map,
                                                         uint32_t* __restrict__ plist, int* __restrict__ pcnt,
                                                         int npairs) {
  const int pair = (int)(blockIdx.x % (unsigned)npairs), bh = (int)(blockIdx.x / (unsigned)npairs), nb = g.nb;
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
  const uint8_t* rb = rows_sm + nb;
  uint32_t* out = plist + ((size_t)bh * npairs + pair) * (2 * nb);
  __shared__ int wtot[8];
  int run = 0;
  int counts[3];
  const int phase_bits[3] = {16, 8, 4};
  for (int ph = 0; ph < 3; ++ph) {
    const int start = run;
    int seen = 0;  // entries of the phase before this chunk
    for (int base = 0; base < nb; base += 256) {
      const int kb = base + threadIdx.x;
      const bool a = kb < nb && ra[kb] == phase_bits[ph], b = kb < nb && rb[kb] == phase_bits[ph];
      const unsigned bal = __ballot_sync(0xffffffffu, a || b);
      if (lane == 0) wtot[warp] = __popc(bal);
      __syncthreads();
      if (a || b) {
        int i = seen + __popc(bal & ((1u << lane) - 1u));
        for (int w = 0; w < warp; ++w) i += wtot[w];
        const int rx = kb % g.nrx, ry = (kb / g.nrx) % g.nry;
        const bool full = (ry + 1) * g.rh <= g.Hh && (rx + 1) * g.rw <= g.Ww;
        out[start + i] = (uint32_t)kb | ((uint32_t)a << 16) | ((uint32_t)b << 17) | ((uint32_t)ph << 18) |
                         ((uint32_t)full << 20);
      }
      for (int w = 0; w < 8; ++w) seen += wtot[w];
      __syncthreads();
    }
    run = start + seen;
    counts[ph] = seen;
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

// bf16 matrix [rows][cols] in boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool map_bf16_rows(CUtensorMap* m, const void* base, uint64_t rows, uint32_t cols, uint32_t box_rows) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Status word of the dense path (its waits are bounded like the sparse
// path's; the dense entry point has no workspace to report through).
__device__ int g_dense_status;

// Kernel attributes: the dynamic shared memory (two tiles of about 110 KB)
// and the largest shared-memory carveout.
template <int D, bool kDense>
cudaError_t configure_tc() {
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, kDense>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Smem<D>::BYTES);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(attn_tc_kernel<D, kDense>, cudaFuncAttributePreferredSharedMemoryCarveout,
                              (int)cudaSharedmemCarveoutMaxShared);
}

template <int D, bool kDense>
cudaError_t launch_tc(const Geom& g, const CUtensorMap* maps, const TcArgs& A, cudaStream_t st) {
  // kTiles query-block pairs per CTA
  const long long ctas = ((long long)A.npairs * g.BH + kTiles - 1) / kTiles;
  if (ctas > 0x7fffffffLL) return cudaErrorNotSupported;
  cudaError_t e = configure_tc<D, kDense>();
  if (e != cudaSuccess) return e;
  attn_tc_kernel<D, kDense><<<(unsigned)ctas, kThreads, Smem<D>::BYTES, st>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], maps[7], maps[8], maps[9], g, A);
  return cudaGetLastError();
}

template <int D, bool kDense>
cudaError_t occupancy_tc(int* ctas_per_sm) {
  cudaError_t e = configure_tc<D, kDense>();
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, attn_tc_kernel<D, kDense>, kThreads,
                                                       Smem<D>::BYTES);
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

cudaError_t launch_pair_lists(const Geom& g, const Layout& L, void* ws, cudaStream_t st) {
  const int npairs = (g.nb + 1) / 2;
  const size_t smem = (2 * (size_t)g.nb + 15) & ~(size_t)15;  // the pair's two map rows
  if (smem > 227 * 1024 || (long long)npairs * g.BH > 0x7fffffffLL) return cudaErrorNotSupported;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(pair_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  pair_lists_kernel<<<(unsigned)((long long)npairs * g.BH), 256, smem, st>>>(
      g, at<uint8_t>(ws, L, R_MAP), at<uint32_t>(ws, L, R_PLIST), at<int>(ws, L, R_PCNT), npairs);
  return cudaGetLastError();
}

cudaError_t launch_attention_tc(const Geom& g, const Layout& L, const void* q, const void* k, const void* v,
                                void* ws, void* out, cudaStream_t st, uint32_t spin, int poison) {
  if (!tma_available()) return cudaErrorNotSupported;
  CUtensorMap m[10];
  const int D = g.d;
  const uint64_t rows64 = (uint64_t)g.BH * g.nb * 64, rowsD = (uint64_t)g.BH * g.nb * D;
  const CUtensorMapSwizzle sw8 = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const CUtensorMapSwizzle sw4 = D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  if (!make_region_map(&m[0], q, g, true) || !make_region_map(&m[1], k, g, true) ||
      !make_region_map(&m[2], v, g, true) || !make_region_map(&m[3], out, g, true) ||
      !map_rows(&m[4], at<int8_t>(ws, L, R_Q_I8), rows64, D, 64, sw8) ||
      !map_rows(&m[5], at<int8_t>(ws, L, R_K_I8), rows64, D, 64, sw8) ||
      !map_bf16_rows(&m[6], at<__nv_bfloat16>(ws, L, R_V_I8), rows64, D, 64) ||
      !map_rows(&m[7], at<uint8_t>(ws, L, R_Q_F4), rows64, D / 2, 64, sw4) ||
      !map_rows(&m[8], at<uint8_t>(ws, L, R_K_F4), rows64, D / 2, 64, sw4) ||
      !map_rows(&m[9], at<uint8_t>(ws, L, R_V_F4), rowsD, 32, D, CU_TENSOR_MAP_SWIZZLE_32B))
    return cudaErrorInvalidValue;
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
  A.status = at<int>(ws, L, R_STATUS);
  A.npairs = (g.nb + 1) / 2;
  A.spin = spin;
  A.poison = poison;
  return D == 128 ? launch_tc<128, false>(g, m, A, st) : launch_tc<64, false>(g, m, A, st);
}

cudaError_t launch_attention(const Geom& g, const Layout& L, const void* q, const void* k, const void* v,
                             void* ws, void* out, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(at<int>(ws, L, R_STATUS), 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  return launch_attention_tc(g, L, q, k, v, ws, out, st, kDefaultSpin, -1);
}

cudaError_t launch_attention_test(const Geom& g, const Layout& L, const void* q, const void* k, const void* v,
                                  void* ws, void* out, cudaStream_t st, uint32_t spin, int poison) {
  cudaError_t e = cudaMemsetAsync(at<int>(ws, L, R_STATUS), 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  return launch_attention_tc(g, L, q, k, v, ws, out, st, spin, poison);
}

// Dense attention on the same kernel: the token axis viewed as one frame of
// 1 x N tokens cut into 64-token regions (natural order), every key block in
// the 16-bit phase, the tail block masked and clipped by TMA like a padded region.
cudaError_t launch_dense(int B, int H, int N, int d, const void* q, const void* k, const void* v, void* out,
                         cudaStream_t st) {
  if (!tma_available() || N < 64 || (d != 64 && d != 128)) return cudaErrorNotSupported;
  Geom g{};
  g.B = B; g.H = H; g.T = 1; g.Hh = 1; g.Ww = N; g.d = d; g.rh = 1; g.rw = 64;
  g.nry = 1; g.nrx = (N + 63) / 64; g.nb = g.nrx; g.N = N; g.BH = B * H;
  CUtensorMap m[10];
  if (!make_region_map(&m[0], q, g, true) || !make_region_map(&m[1], k, g, true) ||
      !make_region_map(&m[2], v, g, true) || !make_region_map(&m[3], out, g, true))
    return cudaErrorInvalidValue;
  for (int i = 4; i < 10; ++i) m[i] = m[0];  // the low-bit tensor maps are never used in dense mode
  int* status = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_dense_status);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(status, 0, sizeof(int), st)) != cudaSuccess) return e;
  TcArgs A{};
  A.status = status;
  A.npairs = (g.nb + 1) / 2;
  A.spin = kDefaultSpin;
  A.poison = -1;
  return d == 128 ? launch_tc<128, true>(g, m, A, st) : launch_tc<64, true>(g, m, A, st);
}

cudaError_t attention_occupancy(int d, bool dense, int* ctas_per_sm) {
  if (d != 64 && d != 128) return cudaErrorInvalidValue;
  if (dense) return d == 128 ? occupancy_tc<128, true>(ctas_per_sm) : occupancy_tc<64, true>(ctas_per_sm);
  return d == 128 ? occupancy_tc<128, false>(ctas_per_sm) : occupancy_tc<64, false>(ctas_per_sm);
}

cudaError_t dense_status(int* word, cudaStream_t st) {
  int* status = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_dense_status);
  if (e == cudaSuccess) e = cudaMemcpyAsync(word, status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return e;
}

}  // namespace da2
