// Stage 3 on the Blackwell tensor cores (tcgen05 + TMEM + TMA).
//
// DraftAttention2 abstract and reading note (Method overview bullet 4): one
// kernel runs a phase per precision for each query block, sharing data
// movement, softmax statistics and one output accumulator.  DraftAttention (v1)
// abstract: the output is restored to the original token order.
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
// Per key block j (warp roles: 4 softmax warps own one TMEM lane / tile row
// each; one TMA producer warp; one MMA warp):
//   16-bit  S = Q·K^T (kind::f16, bf16, M128 N64, fp32 in TMEM, 2 buffers);
//           softmax threads turn their row into P = exp2(s − m_ref) in bf16
//           (m_ref an integer exponent raised lazily: O is rescaled in TMEM, by
//           a power of two, only when the row max grows by more than 2^8) and
//           write it K-major to shared memory;
//           O += P·V (kind::f16, V read MN-major straight from the TMA tile).
//   8-bit   S = Q8·K8^T (kind::i8, s32); P8 = round(255·exp(s − m_blk)) (u8);
//           X = P8·V8^T (kind::i8 u8×s8, s32, 2 buffers); the softmax thread
//           merges X into O in TMEM with exp(m_blk − m)/255 and the channel
//           scales (the phase-boundary rescale of the pages).
//   4-bit   handled by the legacy kernel (not routed here yet).
// Operands arrive by TMA: bf16 Q/K/V as 8×8-token region boxes straight from
// the [B,H,N,d] tensors (padding is the TMA zero fill), INT8 codes as 2-D
// boxes of the workspace.  The epilogue writes O through the same region box
// with a TMA store, whose clipping drops the padding rows — the restore.
// Every mbarrier wait is bounded; on expiry the CTA raises the workspace status
// word and skips ahead to release its tensor memory.
#include <cuda.h>

#include <mutex>

#include "da2_internal.cuh"
#include "sm100.cuh"

namespace da2 {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kThreads = 192;  // warps 0-3 softmax, warp 4 TMA, warp 5 MMA
constexpr int kStages = 3;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// shared-memory map (offsets from a 1024-aligned base)
constexpr uint32_t SM_Q16 = 0;         // [2 halves][128 rows][128 B], SW128
constexpr uint32_t SM_Q8 = 32768;      // [128 rows][128 B], SW128
constexpr uint32_t SM_STAGE = 49152;   // kStages x 32 KB: K at +0, V at +16384
constexpr uint32_t STAGE_BYTES = 32768;
constexpr uint32_t SM_P = SM_STAGE + kStages * STAGE_BYTES;  // 2 x 16 KB
constexpr uint32_t SM_VS = SM_P + 2 * 16384;                 // 128 fp32 V scales
constexpr uint32_t SM_BAR = SM_VS + 512;                     // mbarriers
constexpr uint32_t SM_MISC = SM_BAR + 256;
constexpr uint32_t SM_TOTAL = SM_MISC + 64;
constexpr uint32_t kSmemBytes = SM_TOTAL + 1024;  // + alignment slack

// TMEM columns
constexpr uint32_t TM_O = 0, TM_S = 128, TM_X = 256;  // S: 2 x 64, X: 2 x 128

// mbarrier slots (8 bytes each)
enum {
  B_Q16 = 0, B_Q8, B_KV_FULL, B_KV_EMPTY = B_KV_FULL + kStages, B_S_FULL = B_KV_EMPTY + kStages,
  B_S_FREE = B_S_FULL + 2, B_P_FULL = B_S_FREE + 2, B_P_FREE = B_P_FULL + 2, B_X_FULL = B_P_FREE + 2,
  B_X_FREE = B_X_FULL + 2, B_DONE = B_X_FREE + 2, B_COUNT
};
static_assert(B_COUNT * 8 <= 256, "barrier area");

struct TcArgs {
  const uint32_t* plist;  // [BH][npairs][2*nb]
  const int* pcnt;        // [BH][npairs][4]
  const float* q_s8;
  const float* k_s8;
  const float* v_s8;
  int* status;
  int npairs;
};

__device__ __forceinline__ void raise_timeout(int* status) { atomicOr(status, 1); }

// Items: kb | inA << 16 | inB << 17 | kind << 18 (kind 0 = 16-bit, 1 = 8-bit).
__device__ __forceinline__ int item_kb(uint32_t e) { return (int)(e & 0xffffu); }
__device__ __forceinline__ int item_kind(uint32_t e) { return (int)((e >> 18) & 3u); }

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const __grid_constant__ CUtensorMap tmQ8, const __grid_constant__ CUtensorMap tmK8,
               const __grid_constant__ CUtensorMap tmV8, Geom g, TcArgs A) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s0 = (uint32_t)__cvta_generic_to_shared(smem);
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qa = 2 * pair, qb = (2 * pair + 1 < g.nb) ? 2 * pair + 1 : -1;
  const size_t prow = (size_t)bh * A.npairs + pair;
  const int4 pc = *reinterpret_cast<const int4*>(A.pcnt + prow * 4);
  const int n16 = pc.x, n8 = pc.y;
  const int n = n16 + n8;
  const uint32_t* items = A.plist + prow * (size_t)(2 * g.nb);
  auto bar = [&](int i) { return s0 + SM_BAR + 8u * (uint32_t)i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + SM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM_MISC + 8);

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q16), 1);
    mbar_init(bar(B_Q8), 1);
    for (int s = 0; s < kStages; ++s) { mbar_init(bar(B_KV_FULL + s), 1); mbar_init(bar(B_KV_EMPTY + s), 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_S_FULL + b), 1);
      mbar_init(bar(B_S_FREE + b), 4);
      mbar_init(bar(B_P_FULL + b), 4);
      mbar_init(bar(B_P_FREE + b), 1);
      mbar_init(bar(B_X_FULL + b), 1);
      mbar_init(bar(B_X_FREE + b), 4);
    }
    mbar_init(bar(B_DONE), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc(s0 + SM_MISC, 512);
  if (threadIdx.x < kD) reinterpret_cast<float*>(smem + SM_VS)[threadIdx.x] = A.v_s8[(size_t)bh * kD + threadIdx.x];
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

  if (warp == 4) {
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
      for (int j = 0; j < n; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !mbar_wait(bar(B_KV_EMPTY + s), ((j / kStages) - 1) & 1)) {
          raise_timeout(A.status); *abort_flag = 1; break;
        }
        const uint32_t e = items[j];
        const int kb = item_kb(e);
        const uint32_t st = s0 + SM_STAGE + s * STAGE_BYTES;
        if (item_kind(e) == 0) {
          mbar_expect_tx(bar(B_KV_FULL + s), 32768u);
          box(kb, cx, cy, cf);
          tma_load_4d(st, &tmK, bar(B_KV_FULL + s), 0, cx, cy, cf);
          tma_load_4d(st + 8192, &tmK, bar(B_KV_FULL + s), 64, cx, cy, cf);
          tma_load_4d(st + 16384, &tmV, bar(B_KV_FULL + s), 0, cx, cy, cf);
          tma_load_4d(st + 16384 + 8192, &tmV, bar(B_KV_FULL + s), 64, cx, cy, cf);
        } else {
          mbar_expect_tx(bar(B_KV_FULL + s), 16384u);
          tma_load_2d(st, &tmK8, bar(B_KV_FULL + s), 0, (bh * g.nb + kb) * 64);
          tma_load_2d(st + 16384, &tmV8, bar(B_KV_FULL + s), 0, (bh * g.nb + kb) * kD);
        }
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      const uint32_t id16 = idesc(kDF32, kFmtBF16, kFmtBF16, false, false, 128, 64);
      const uint32_t idpv = idesc(kDF32, kFmtBF16, kFmtBF16, false, true, 128, 128);
      const uint32_t id8 = idesc(kDS32, kFmtS8, kFmtS8, false, false, 128, 64);
      const uint32_t idx8 = idesc(kDS32, kFmtU8, kFmtS8, false, false, 128, 128);
      bool ok = true;
      if (n16 > 0) ok = ok && mbar_wait(bar(B_Q16), 0);
      if (n8 > 0) ok = ok && mbar_wait(bar(B_Q8), 0);
      int x_uses = 0;
      auto issue_pv = [&](int i) -> bool {
        const uint32_t e = items[i];
        const int b = i & 1, s = i % kStages;
        if (!mbar_wait(bar(B_P_FULL + b), (i >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t st = s0 + SM_STAGE + s * STAGE_BYTES;
        const uint32_t pb = s0 + SM_P + b * 16384;
        if (item_kind(e) == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tbase + TM_O, smem_desc(pb + kk * 32, 16, 1024, SW_128),
                    smem_desc(st + 16384 + kk * 2048, 8192, 1024, SW_128), idpv, 1u);
        } else {
          const int xb = x_uses & 1;
          if (x_uses >= 2 && !mbar_wait(bar(B_X_FREE + xb), ((x_uses >> 1) - 1) & 1)) return false;
          tc_fence_after();
          const uint32_t xt = tbase + TM_X + xb * 128;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_i8(xt, smem_desc(pb + kk * 32, 16, 512, SW_64), smem_desc(st + 16384 + kk * 32, 16, 512, SW_64),
                   idx8, kk > 0 ? 1u : 0u);
          mma_commit(bar(B_X_FULL + xb));
          ++x_uses;
        }
        mma_commit(bar(B_P_FREE + b));
        mma_commit(bar(B_KV_EMPTY + s));
        return true;
      };
      for (int j = 0; ok && j < n; ++j) {
        const uint32_t e = items[j];
        const int s = j % kStages, b = j & 1;
        if (!mbar_wait(bar(B_KV_FULL + s), (j / kStages) & 1)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(bar(B_S_FREE + b), ((j >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = s0 + SM_STAGE + s * STAGE_BYTES;
        const uint32_t sd = tbase + TM_S + b * 64;
        if (item_kind(e) == 0) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int h = k >> 2, kk = k & 3;
            mma_f16(sd, smem_desc(s0 + SM_Q16 + h * 16384 + kk * 32, 16, 1024, SW_128),
                    smem_desc(st + h * 8192 + kk * 32, 16, 1024, SW_128), id16, k > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8(sd, smem_desc(s0 + SM_Q8 + kk * 32, 16, 1024, SW_128),
                   smem_desc(st + kk * 32, 16, 1024, SW_128), id8, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(B_S_FULL + b));
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && n > 0) ok = issue_pv(n - 1);
      mma_commit(bar(B_DONE));
      if (!ok) { raise_timeout(A.status); *abort_flag = 1; }
    }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-3
    const int row = threadIdx.x;  // TMEM lane and tile row
    const bool in_b = row >= 64;
    const int qrow_blk = in_b ? qb : qa;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float sl2 = kLog2e * rsqrtf((float)kD);
    const float sq = (n8 > 0 && qrow_blk >= 0) ? A.q_s8[(size_t)bh * g.nb + qrow_blk] : 0.f;
    const float* vs = reinterpret_cast<const float*>(smem + SM_VS);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    {  // O starts at zero
      uint32_t z[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
      for (int c = 0; c < 128; c += 32) tmem_st32(tbase + lane_off + TM_O + c, z);
      tmem_wait_st();
    }
    int x_uses = 0;
    // INT8 block results are merged one INT8 item late, so that X of item i is
    // computed while the softmax of the next item runs.
    bool have_pend = false, pend_member = false;
    float pend_mb = 0.f, pend_lb = 0.f;
    auto merge_x = [&]() -> bool {
      const int xb = x_uses & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_X_FULL + xb), (x_uses >> 1) & 1))) return false;
      tc_fence_after();
      if (pend_member) {
        const float mn = fmaxf(m_ref, pend_mb);
        const float ao = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - mn);
        const float ab = fast_exp2(pend_mb - mn);
        const float f = ab * (1.0f / 255.0f);
        l = l * ao + pend_lb * ab;
        m_ref = mn;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t xr[32], orr[32];
          tmem_ld32(tbase + lane_off + TM_X + xb * 128 + c, xr);
          tmem_ld32(tbase + lane_off + TM_O + c, orr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float o = __uint_as_float(orr[i]) * ao + f * vs[c + i] * (float)(int)xr[i];
            orr[i] = __float_as_uint(o);
          }
          tmem_st32(tbase + lane_off + TM_O + c, orr);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_X_FREE + xb));
      ++x_uses;
      have_pend = false;
      return true;
    };

    for (int j = 0; ok && j < n; ++j) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
      const uint32_t e = items[j];
      const int kb = item_kb(e), kind = item_kind(e);
      const bool member = ((e >> (in_b ? 17 : 16)) & 1u) != 0;
      const int b = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + b), (j >> 1) & 1))) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tbase + lane_off + TM_S + b * 64, sr);
      tmem_ld32(tbase + lane_off + TM_S + b * 64 + 32, sr + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_S_FREE + b));

      // real-key mask of the key block
      unsigned long long vmask;
      {
        const int rx = kb % g.nrx, ry = (kb / g.nrx) % g.nry;
        const int vy = min(g.rh, g.Hh - ry * g.rh), vx = min(g.rw, g.Ww - rx * g.rw);
        const unsigned long long rowbits = (vx >= 64) ? ~0ull : ((1ull << vx) - 1ull);
        vmask = 0;
        for (int i = 0; i < vy; ++i) vmask |= rowbits << (g.rw * i);
      }
      float mb = -INFINITY, lb = 0.f;
      uint32_t pw[32];  // packed P row: 32 x bf16x2 (16-bit) or 16 x u8x4 (8-bit)
      if (kind == 0) {
        if (member) {
          float mx = -INFINITY;
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const float v = ((vmask >> i) & 1ull) ? __uint_as_float(sr[i]) * sl2 : -INFINITY;
            sr[i] = __float_as_uint(v);
            mx = fmaxf(mx, v);
          }
          // raise the reference lazily; the O rescale is warp-collective (TMEM
          // access), so a warp rescales when any of its rows needs it
          const bool need = mx > m_ref + kRescaleThreshold || m_ref == -INFINITY;
          const bool need_o = need && m_ref != -INFINITY;
          if (__any_sync(0xffffffffu, need_o)) {
            bool w_ok = j < 1 || mbar_wait(bar(B_P_FREE + ((j - 1) & 1)), ((j - 1) >> 1) & 1);
            if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
            tc_fence_after();
            // the reference is an integer exponent, so the factor is a power of two
            const float a = need_o ? ldexpf(1.0f, (int)(m_ref - ceilf(mx))) : 1.0f;
#pragma unroll 1
            for (int c = 0; c < 128; c += 32) {
              uint32_t orr[32];
              tmem_ld32(tbase + lane_off + TM_O + c, orr);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * a);
              tmem_st32(tbase + lane_off + TM_O + c, orr);
            }
            tmem_wait_st();
            l *= a;
          }
          // P is exp2(s - m_ref) with m_ref = an integer >= max - 8: its bf16
          // rounding is the same as relative to 2^ceil(row max), whatever the
          // reference, since bf16 rounding commutes with powers of two
          if (need) m_ref = ceilf(mx);
          float sum = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p0 = fast_exp2(__uint_as_float(sr[2 * i]) - m_ref);
            const float p1 = fast_exp2(__uint_as_float(sr[2 * i + 1]) - m_ref);
            sum += p0 + p1;
            __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
            pw[i] = *reinterpret_cast<uint32_t*>(&h);
          }
          l += sum;
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) pw[i] = 0u;
        }
      } else {
        if (member) {
          const float sc = sq * A.k_s8[(size_t)bh * g.nb + kb] * sl2;
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const float v = ((vmask >> i) & 1ull) ? (float)(int)sr[i] * sc : -INFINITY;
            sr[i] = __float_as_uint(v);
            mb = fmaxf(mb, v);
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            uint32_t w = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float p = fast_exp2(__uint_as_float(sr[4 * i + q]) - mb);
              lb += p;
              w |= (__float2uint_rn(255.f * p) & 0xffu) << (8 * q);
            }
            pw[i] = w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pw[i] = 0u;
        }
      }
      // P buffer b is free once the P·V of item j-2 completed
      if (!__all_sync(0xffffffffu, j < 2 || mbar_wait(bar(B_P_FREE + b), ((j >> 1) - 1) & 1))) { ok = false; break; }
      uint8_t* pb = smem + SM_P + b * 16384;
      if (kind == 0) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(pb + row * 128 + ((c ^ (row & 7)) * 16)) =
              make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(pb + row * 64 + ((c ^ ((row >> 1) & 3)) * 16)) =
              make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P_FULL + b));
      if (kind == 1) {
        if (have_pend && !merge_x()) { ok = false; break; }
        have_pend = true;
        pend_member = member;
        pend_mb = mb;
        pend_lb = lb;
      }
    }
    if (ok && have_pend) ok = merge_x();
    // wait for every MMA, then the epilogue
    if (ok && !__all_sync(0xffffffffu, mbar_wait(bar(B_DONE), 0))) ok = false;
    tc_fence_after();
    if (!ok) { raise_timeout(A.status); *abort_flag = 1; }
    // O row / l → bf16 → shared tile (reusing Q16's area, same SW128 layout) → TMA store
    {
      const float il = (l > 0.f) ? 1.0f / l : 0.f;
      uint8_t* ot = smem + SM_Q16;
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        uint32_t orr[32];
        tmem_ld32(tbase + lane_off + TM_O + c, orr);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(orr[2 * i]) * il,
                                                   __uint_as_float(orr[2 * i + 1]) * il);
          w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        const int half = c >> 6, ch0 = (c & 63) >> 3;  // 16-byte chunk index within the half
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = ch0 + q;
          *reinterpret_cast<uint4*>(ot + half * 16384 + row * 128 + ((chunk ^ (row & 7)) * 16)) =
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
  if (warp == 5) {
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
// ascending key blocks either member keeps in that phase, with member flags.
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
        out[off] = (uint32_t)kb | ((uint32_t)a << 16) | ((uint32_t)b << 17) | ((uint32_t)ph << 18);
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
  return g.d == kD && g.n4 == 0 && encode_fn() != nullptr;
}

cudaError_t launch_pair_lists(const Geom& g, const Layout& L, void* ws, cudaStream_t st) {
  const int npairs = (g.nb + 1) / 2;
  pair_lists_kernel<<<dim3(npairs, g.BH), 256, 0, st>>>(g, at<uint8_t>(ws, L, R_MAP), at<uint32_t>(ws, L, R_PLIST),
                                                       at<int>(ws, L, R_PCNT), npairs);
  return cudaGetLastError();
}

cudaError_t launch_attention_tc(const Geom& g, const Layout& L, const void* q, const void* k, const void* v,
                                void* ws, void* out, cudaStream_t st) {
  CUtensorMap tq, tk, tv, to, tq8, tk8, tv8;
  const uint64_t rows64 = (uint64_t)g.BH * g.nb * 64, rows128 = (uint64_t)g.BH * g.nb * kD;
  if (!map_regions(&tq, q, g) || !map_regions(&tk, k, g) || !map_regions(&tv, v, g) || !map_regions(&to, out, g) ||
      !map_rows(&tq8, at<int8_t>(ws, L, R_Q_I8), rows64, kD, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map_rows(&tk8, at<int8_t>(ws, L, R_K_I8), rows64, kD, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map_rows(&tv8, at<int8_t>(ws, L, R_V_I8), rows128, 64, kD, CU_TENSOR_MAP_SWIZZLE_64B))
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
  A.status = status;
  A.npairs = (g.nb + 1) / 2;
  e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<<<dim3(A.npairs, g.BH), kThreads, kSmemBytes, st>>>(tq, tk, tv, to, tq8, tk8, tv8, g, A);
  return cudaGetLastError();
}

}  // namespace da2
