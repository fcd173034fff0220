// Internal definitions shared by the libda2 translation units: problem
// geometry, workspace layout and small device helpers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/da2.h"

namespace da2 {

constexpr int kBlockTokens = 64;     // one region = one 64-token block
constexpr int kRankPasses = 8;       // 64-bit ranking key, 8 bits per pass
constexpr int kTargets = 3;          // rank cuts: n16, n16+n8, n16+n8+n4

// NVFP4 e4m3 scales are stored in the layout the tensor core reads them from
// (tcgen05.cp 32x128b.warpx4): per 64-element chunk of the reduction axis, an
// atom of 32 lines x 16 bytes in which line i holds the 4 scales (one per 16
// elements) of rows i, i+32, i+64, i+96 as four 32-bit words.  A 64-row Q/K
// block fills words 0 and 1 of each line and repeats them in words 2 and 3.
constexpr int kSfAtomBytes = 512;
__host__ __device__ __forceinline__ int sf_atom_offset(int row, int mb) {
  return (mb >> 2) * kSfAtomBytes + (row & 31) * 16 + (row >> 5) * 4 + (mb & 3);
}

// Geometry of one problem, derived once on the host and passed by value.
struct Geom {
  int B, H, T, Hh, Ww, d, rh, rw;
  int nry, nrx, nb, N;
  int BH;
  float lambda;
  long long n16, n8, n4;       // per head
  long long cut[kTargets];     // cumulative counts n16, n16+n8, n16+n8+n4
};

// Workspace: byte offsets of every region, each 256-byte aligned.
enum Region {
  R_STATUS = 0, R_PERM,
  R_Q_AVG, R_K_AVG, R_Q_MAX, R_K_MAX,
  R_Q_I8, R_K_I8, R_Q_S8, R_K_S8,
  R_Q_F4, R_K_F4, R_Q_SF4, R_K_SF4,
  R_V_I8, R_V_S8, R_V_F4, R_V_SF4, R_V_G4,
  R_SCORES, R_MAP, R_LISTS, R_COUNTS,
  R_V_AMAX, R_LOGB, R_HIST, R_RSTATE,
  R_PLIST, R_PCNT,
  R_COUNT_
};

struct Layout {
  size_t off[R_COUNT_];
  size_t size[R_COUNT_];
  size_t total;
};

// Per-(head, target) radix-select state.
struct RankState {
  unsigned long long prefix;   // key bits fixed so far (high bits first)
  long long remaining;         // rank still to skip inside the prefix's bucket
  long long count;             // the cut (number of pairs inside); 0 = empty cut
  unsigned long long thresh;   // final key threshold: pair inside iff key >= thresh
  int done;                    // 1 once thresh is final
  int pad;
};

inline Layout make_layout(const Geom& g) {
  Layout L{};
  const size_t bh = (size_t)g.BH, nb = (size_t)g.nb, d = (size_t)g.d, S = kBlockTokens;
  L.size[R_STATUS] = 256;
  L.size[R_PERM] = nb * S * 4;
  L.size[R_Q_AVG] = L.size[R_K_AVG] = L.size[R_Q_MAX] = L.size[R_K_MAX] = bh * nb * d * 4;
  L.size[R_Q_I8] = L.size[R_K_I8] = bh * nb * S * d;
  L.size[R_Q_S8] = L.size[R_K_S8] = bh * nb * 4;
  L.size[R_Q_F4] = L.size[R_K_F4] = bh * nb * S * d / 2;
  L.size[R_Q_SF4] = L.size[R_K_SF4] = bh * nb * (d / 64) * kSfAtomBytes;
  L.size[R_V_I8] = bh * nb * S * d * 2;  // INT8 codes held as bf16 values, [slot][channel] per block
  L.size[R_V_S8] = bh * d * 4;
  L.size[R_V_F4] = bh * nb * d * S / 2;
  L.size[R_V_SF4] = bh * nb * kSfAtomBytes;
  L.size[R_V_G4] = bh * d * 4;
  L.size[R_SCORES] = bh * nb * nb * 4;
  L.size[R_MAP] = bh * nb * nb;
  L.size[R_LISTS] = bh * nb * nb * 2;
  L.size[R_COUNTS] = bh * nb * 4 * 4;
  L.size[R_V_AMAX] = bh * d * 4 + (bh + 1) * 4;  // absmax bits, work counter, done counter per head
  L.size[R_LOGB] = bh * nb * nb * 4;
  L.size[R_HIST] = (size_t)kRankPasses * bh * kTargets * 256 * 4;
  L.size[R_RSTATE] = bh * kTargets * sizeof(RankState);
  // merged key lists of query-block pairs (2p, 2p+1): at most 2*nb entries each
  L.size[R_PLIST] = bh * ((nb + 1) / 2) * (2 * nb) * 4;
  L.size[R_PCNT] = bh * ((nb + 1) / 2) * 4 * 4;
  size_t o = 0;
  for (int r = 0; r < R_COUNT_; ++r) {
    L.off[r] = o;
    o += (L.size[r] + 255) & ~(size_t)255;
  }
  L.total = o;
  return L;
}

template <typename T>
inline T* at(void* ws, const Layout& L, Region r) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + L.off[r]);
}

// ---------------------------------------------------------------- device side

// Token index of slot `s` of block `blk`, or -1 for a padding slot.
__host__ __device__ __forceinline__ int slot_token(const Geom& g, int blk, int s) {
  const int rx = blk % g.nrx;
  const int tmp = blk / g.nrx;
  const int ry = tmp % g.nry;
  const int t = tmp / g.nry;
  const int i = s / g.rw, j = s - (s / g.rw) * g.rw;
  const int y = ry * g.rh + i, x = rx * g.rw + j;
  if (y >= g.Hh || x >= g.Ww) return -1;
  return (t * g.Hh + y) * g.Ww + x;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Hardware conversions (PTX cvt, round-to-nearest-even, saturate to finite).
// Two fp32 → e4m3x2: `hi` goes to the upper byte.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// Two fp32 → e2m1x2 in one byte: `hi` goes to the upper nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// e4m3 byte → fp32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  uint32_t h2;
  uint16_t b = (uint16_t)(byte & 0xff);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(b));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffff)));
}
// Packed e2m1x2 byte → f16x2 (low nibble → low half), exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t h2;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h2) : "r"(byte));
  return h2;
}

// 2^x on the SFU (MUFU.EX2), flushing denormal results to zero.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// fp32 → key whose unsigned order is the float order (-0 canonicalised to +0).
__device__ __forceinline__ uint32_t float_order_key(float f) {
  uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace da2

// Launchers implemented in the .cu files (all asynchronous on `st`).
namespace da2 {
cudaError_t launch_prepare(const Geom& g, const Layout& L, const void* q, const void* k,
                           const void* v, void* ws, cudaStream_t st);
cudaError_t launch_draft(const Geom& g, const Layout& L, void* ws, cudaStream_t st);
cudaError_t launch_rank(const Geom& g, const Layout& L, void* ws, bool hist0_done,
                        cudaStream_t st);
cudaError_t launch_attention(const Geom& g, const Layout& L, const void* q, const void* k,
                             const void* v, void* ws, void* out, cudaStream_t st);
cudaError_t launch_dense(int B, int H, int N, int d, const void* q, const void* k,
                         const void* v, void* out, cudaStream_t st);
// Status word of the dense path: synchronises `st` and copies it to *word.
// CTAs of the attention kernel (head dimension d, sparse or dense) an SM holds at once.
cudaError_t attention_occupancy(int d, bool dense, int* ctas_per_sm);
cudaError_t dense_status(int* word, cudaStream_t st);
cudaError_t launch_pair_lists(const Geom& g, const Layout& L, void* ws, cudaStream_t st);
// TMA: whether the driver's tensor-map encoder was found, and the 4-D view
// [B*H*T][Hh][Ww][d] of a bf16 [B,H,N,d] tensor in {64 channels, rw, rh, 1}
// region boxes (zero fill outside the frame).
bool tma_available();
bool make_region_map(CUtensorMap* m, const void* base, const Geom& g, bool swizzle128);
// The attention kernel with an explicit wait bound (polls) and a CTA whose
// first key load is withheld (-1: none), for the failure-path test.
cudaError_t launch_attention_test(const Geom& g, const Layout& L, const void* q, const void* k,
                                  const void* v, void* ws, void* out, cudaStream_t st,
                                  uint32_t spin, int poison);
cudaError_t launch_rank_noalloc(const Geom& g, const float* scores, uint8_t* map, uint16_t* lists,
                                int* counts, cudaStream_t st);
}  // namespace da2
