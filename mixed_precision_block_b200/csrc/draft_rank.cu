// Stage 2: draft attention map, shared per-head ranking, precision assignment.
//
// DraftAttention2 abstract; reading note Method overview bullets 1-2 and
// Figure 2.  The map D = (1-lambda) softmax(avgQ avgK^T/sqrt d)
//                     + lambda softmax(maxQ maxK^T/sqrt d)
// is built per head over region pairs; one ranking per head (descending D,
// ties by ascending pair index) hands out 16-bit, then INT8, then NVFP4, and
// the rest of the pairs are skipped.
//
// draft_logits   fp32 SIMT GEMM tiles (128x128, 8x8 per thread) → raw logits of both maps
// draft_mix      one CTA per query region: row softmaxes, the mix, and the
//                first radix-select histogram of the ranking keys
// rank_*         MSD radix select, 8 bits per pass, of the three cut keys on
//                the 64-bit key (order(D) << 32 | ~pair): a pass only counts
//                keys that still match a cut's prefix, and a cut finishes as
//                soon as its rank is the last one in its bucket
// rank_assign    one CTA per query region: precision per pair, the u8 map and
//                the per-query-block key lists (ballot/popc compaction)
#include <mutex>

#include <cuda.h>

#include "da2_internal.cuh"

namespace da2 {
namespace {


// Logit tiles of 128 x 128 region pairs, both maps one after the other: 256
// threads, each 8 x 8 outputs (rows ty*4.. and 64+ty*4.., columns tx*4.. and
// 64+tx*4..), so a k step is four 16-byte shared loads for 64 FMAs.
constexpr int kLT = 128, kLK = 16;
__global__ void __launch_bounds__(256, 2) draft_logits_kernel(Geom g, const float* __restrict__ qa,
                                                           const float* __restrict__ ka,
                                                           const float* __restrict__ qm,
                                                           const float* __restrict__ km,
                                                           float* __restrict__ la,
                                                           float* __restrict__ lb) {
  const int D = g.d, nb = g.nb;
  const int bh = blockIdx.z;
  const int r0 = blockIdx.y * kLT, c0 = blockIdx.x * kLT;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  __shared__ __align__(16) float sA[2][kLK][kLT];  // [buffer][k][row]
  __shared__ __align__(16) float sB[2][kLK][kLT];  // [buffer][k][col]
  const size_t base = (size_t)bh * nb * D;
  const float sc = 1.0f / sqrtf((float)D);
  const bool vec_out = (nb & 3) == 0;
  const int nk = D / kLK;
#pragma unroll 1
  for (int m = 0; m < 2; ++m) {
    const float* __restrict__ A = m ? qm : qa;
    const float* __restrict__ B = m ? km : ka;
    float* __restrict__ O = m ? lb : la;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    // 128 rows x 16 k of A and of B per chunk: 512 float4 each, two per
    // thread, fetched into registers one chunk ahead of the shared tiles
    float4 av[2], bv[2];
    auto fetch = [&](int k0) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int e = tid + 256 * t, r = e >> 2, kq = e & 3;
        const int gr = r0 + r, gc = c0 + r;
        av[t] = gr < nb ? *reinterpret_cast<const float4*>(A + base + (size_t)gr * D + k0 + 4 * kq)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        bv[t] = gc < nb ? *reinterpret_cast<const float4*>(B + base + (size_t)gc * D + k0 + 4 * kq)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    auto stash = [&](int buf) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int e = tid + 256 * t, r = e >> 2, kq = e & 3;
        sA[buf][4 * kq][r] = av[t].x; sA[buf][4 * kq + 1][r] = av[t].y;
        sA[buf][4 * kq + 2][r] = av[t].z; sA[buf][4 * kq + 3][r] = av[t].w;
        sB[buf][4 * kq][r] = bv[t].x; sB[buf][4 * kq + 1][r] = bv[t].y;
        sB[buf][4 * kq + 2][r] = bv[t].z; sB[buf][4 * kq + 3][r] = bv[t].w;
      }
    };
    fetch(0);
    stash(0);
    __syncthreads();
#pragma unroll 1
    for (int kc = 0; kc < nk; ++kc) {
      const int buf = kc & 1;
      if (kc + 1 < nk) fetch((kc + 1) * kLK);
#pragma unroll
      for (int kk = 0; kk < kLK; ++kk) {
        const float4 a0 = *reinterpret_cast<const float4*>(&sA[buf][kk][ty * 4]);
        const float4 a1 = *reinterpret_cast<const float4*>(&sA[buf][kk][64 + ty * 4]);
        const float4 b0 = *reinterpret_cast<const float4*>(&sB[buf][kk][tx * 4]);
        const float4 b1 = *reinterpret_cast<const float4*>(&sB[buf][kk][64 + tx * 4]);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      if (kc + 1 < nk) stash(buf ^ 1);
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = r0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
      if (r >= nb) continue;
      float* __restrict__ orow = O + ((size_t)bh * nb + r) * nb;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = c0 + 64 * h + tx * 4;
        const float v0 = acc[i][4 * h] * sc, v1 = acc[i][4 * h + 1] * sc;
        const float v2 = acc[i][4 * h + 2] * sc, v3 = acc[i][4 * h + 3] * sc;
        if (vec_out && c + 3 < nb) {
          *reinterpret_cast<float4*>(orow + c) = make_float4(v0, v1, v2, v3);
        } else {
          if (c < nb) orow[c] = v0;
          if (c + 1 < nb) orow[c + 1] = v1;
          if (c + 2 < nb) orow[c + 2] = v2;
          if (c + 3 < nb) orow[c + 3] = v3;
        }
      }
    }
  }
}

__device__ __forceinline__ void online_merge(float& m, float& s, float m2, float s2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;
  s = s * expf(m - mn) + s2 * expf(m2 - mn);
  m = mn;
}

// Block-wide (max, sum-exp) merge over 256 threads.
__device__ __forceinline__ void block_softmax_stats(float& m, float& s, float* sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    online_merge(m, s, m2, s2);
  }
  if (lane == 0) { sm[2 * warp] = m; sm[2 * warp + 1] = s; }
  __syncthreads();
  m = sm[0]; s = sm[1];
  for (int w = 1; w < 8; ++w) online_merge(m, s, sm[2 * w], sm[2 * w + 1]);
  __syncthreads();
}

__device__ __forceinline__ unsigned long long pair_key(float dval, unsigned int pair) {
  return ((unsigned long long)float_order_key(dval) << 32) | (unsigned long long)(0xffffffffu - pair);
}

// One CTA per (query region, head): mix the two row softmaxes into D.
__global__ void __launch_bounds__(256) draft_mix_kernel(Geom g, float* __restrict__ la,
                                                        const float* __restrict__ lb,
                                                        unsigned int* __restrict__ hist0) {
  const int row = blockIdx.x, bh = blockIdx.y, nb = g.nb;
  const size_t o = ((size_t)bh * nb + row) * nb;
  float ma = -INFINITY, sa = 0.f, mb = -INFINITY, sb = 0.f;
  for (int c = threadIdx.x; c < nb; c += 256) {
    online_merge(ma, sa, la[o + c], 1.f);
    online_merge(mb, sb, lb[o + c], 1.f);
  }
  __shared__ float sm[16];
  __shared__ unsigned int h[8][256];
  for (int i = threadIdx.x; i < 8 * 256; i += 256) (&h[0][0])[i] = 0;
  block_softmax_stats(ma, sa, sm);
  block_softmax_stats(mb, sb, sm);
  const float wa = (1.0f - g.lambda) / sa, wb = g.lambda / sb;
  const int warp = threadIdx.x >> 5;
  for (int c = threadIdx.x; c < nb; c += 256) {
    const float dv = wa * expf(la[o + c] - ma) + wb * expf(lb[o + c] - mb);
    la[o + c] = dv;
    const unsigned long long key = pair_key(dv, (unsigned)(row * nb + c));
    atomicAdd(&h[warp][key >> 56], 1u);
  }
  __syncthreads();
  unsigned int* dst = hist0 + (size_t)bh * kTargets * 256;
  for (int b = threadIdx.x; b < 256; b += 256) {
    unsigned int t = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += h[w][b];
    if (t) atomicAdd(dst + b, t);
  }
}

__global__ void rank_init_kernel(Geom g, RankState* st) {
  const int bh = blockIdx.x, t = threadIdx.x;
  if (t >= kTargets) return;
  const long long P = (long long)g.nb * g.nb;
  RankState s{};
  s.count = g.cut[t];
  s.prefix = 0;
  if (s.count == 0 || s.count == P) {
    s.done = 1;
    s.thresh = 0;  // count==P: every key is >= 0; count==0: `count` alone excludes all
  } else {
    s.done = 0;
    s.remaining = s.count - 1;
  }
  st[bh * kTargets + t] = s;
}

// Histogram of digit `pass` over keys that still match each open cut's prefix.
__global__ void __launch_bounds__(256) rank_hist_kernel(Geom g, const float* __restrict__ scores,
                                                        const RankState* __restrict__ st,
                                                        unsigned int* __restrict__ hist, int pass,
                                                        int per_cta) {
  const int bh = blockIdx.y;
  const RankState* s = st + bh * kTargets;
  bool open[kTargets];
  unsigned long long pre[kTargets];
  const int hi_shift = 64 - 8 * pass;  // bits above the digit
  bool any = false;
#pragma unroll
  for (int t = 0; t < kTargets; ++t) {
    open[t] = !s[t].done;
    pre[t] = pass == 0 ? 0ull : (s[t].prefix >> hi_shift);
    any |= open[t];
  }
  if (!any) return;
  __shared__ unsigned int h[kTargets][256];
  for (int i = threadIdx.x; i < kTargets * 256; i += 256) (&h[0][0])[i] = 0;
  __syncthreads();
  const long long P = (long long)g.nb * g.nb;
  const long long p0 = (long long)blockIdx.x * per_cta;
  const long long p1 = min(P, p0 + per_cta);
  const float* sc = scores + (size_t)bh * P;
  const int dshift = 56 - 8 * pass;
  for (long long p = p0 + threadIdx.x; p < p1; p += 256) {
    const unsigned long long key = pair_key(sc[p], (unsigned)p);
    const unsigned long long top = pass == 0 ? 0ull : (key >> hi_shift);
    const unsigned int dig = (unsigned)(key >> dshift) & 255u;
    if (pass == 0) {
      atomicAdd(&h[0][dig], 1u);  // every key, shared by all cuts
    } else {
#pragma unroll
      for (int t = 0; t < kTargets; ++t)
        if (open[t] && top == pre[t]) atomicAdd(&h[t][dig], 1u);
    }
  }
  __syncthreads();
  unsigned int* dst = hist + ((size_t)pass * g.BH + bh) * kTargets * 256;
  for (int i = threadIdx.x; i < kTargets * 256; i += 256) {
    const unsigned int v = (&h[0][0])[i];
    if (v) atomicAdd(dst + i, v);
  }
}

// Pick each open cut's bucket at digit `pass`.  Pass 0's histogram is shared.
__global__ void rank_select_kernel(Geom g, RankState* st, const unsigned int* __restrict__ hist,
                                   int pass, int shared0) {
  const int bh = blockIdx.x, t = threadIdx.x;
  if (t >= kTargets) return;
  RankState s = st[bh * kTargets + t];
  if (s.done) return;
  const unsigned int* h =
      hist + ((size_t)pass * g.BH + bh) * kTargets * 256 + (shared0 ? 0 : t * 256);
  const int dshift = 56 - 8 * pass;
  long long cum = 0;
  for (int b = 255; b >= 0; --b) {
    const long long c = h[b];
    if (cum + c > s.remaining) {
      s.remaining -= cum;
      s.prefix |= (unsigned long long)b << dshift;
      if (s.remaining == c - 1 || pass == kRankPasses - 1) {
        // the cut's rank is the last key of this bucket: every key of the
        // bucket is inside, every key below it is outside
        s.done = 1;
        s.thresh = s.prefix;
      }
      break;
    }
    cum += c;
  }
  st[bh * kTargets + t] = s;
}

__device__ __forceinline__ int precision_of(unsigned long long key, const RankState* s) {
  if (s[0].count > 0 && key >= s[0].thresh) return 16;
  if (s[1].count > 0 && key >= s[1].thresh) return 8;
  if (s[2].count > 0 && key >= s[2].thresh) return 4;
  return 0;
}

__global__ void __launch_bounds__(256) rank_assign_kernel(Geom g, const float* __restrict__ scores,
                                                          const RankState* __restrict__ st,
                                                          uint8_t* __restrict__ map,
                                                          uint16_t* __restrict__ lists,
                                                          int* __restrict__ counts) {
  const int row = blockIdx.x, bh = blockIdx.y, nb = g.nb;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ RankState s[kTargets];
  __shared__ int wtot[8][3];
  __shared__ int total[3];
  if (threadIdx.x < kTargets) s[threadIdx.x] = st[bh * kTargets + threadIdx.x];
  if (threadIdx.x < 3) total[threadIdx.x] = 0;
  __syncthreads();
  const size_t o = ((size_t)bh * nb + row) * nb;
  const unsigned int pbase = (unsigned)row * nb;
  const unsigned lt = (1u << lane) - 1u;
  // pass 1: precision map and list lengths
  int cnt[3] = {0, 0, 0};
  for (int c = threadIdx.x; c < nb; c += 256) {
    const int pr = precision_of(pair_key(scores[o + c], pbase + c), s);
    map[o + c] = (uint8_t)pr;
    cnt[0] += pr == 16; cnt[1] += pr == 8; cnt[2] += pr == 4;
  }
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    int v = cnt[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) atomicAdd(&total[i], v);
  }
  __syncthreads();
  const int c16 = total[0], c8 = total[1], c4 = total[2];
  if (threadIdx.x == 0) {
    int4 w = make_int4(c16, c8, c4, 0);
    *reinterpret_cast<int4*>(counts + ((size_t)bh * nb + row) * 4) = w;
  }
  // pass 2: ordered compaction into [16-list | 8-list | 4-list]
  int run[3] = {0, c16, c16 + c8};
  uint16_t* L = lists + o;
  for (int base = 0; base < nb; base += 256) {
    const int c = base + threadIdx.x;
    int pr = -1;
    if (c < nb) pr = map[o + c];
    unsigned bal[3];
    bal[0] = __ballot_sync(0xffffffffu, pr == 16);
    bal[1] = __ballot_sync(0xffffffffu, pr == 8);
    bal[2] = __ballot_sync(0xffffffffu, pr == 4);
    if (lane == 0)
#pragma unroll
      for (int i = 0; i < 3; ++i) wtot[warp][i] = __popc(bal[i]);
    __syncthreads();
    const int i = pr == 16 ? 0 : pr == 8 ? 1 : pr == 4 ? 2 : -1;
    if (i >= 0) {
      int off = run[i];
      for (int w = 0; w < warp; ++w) off += wtot[w][i];
      L[off + __popc(bal[i] & lt)] = (uint16_t)c;
    }
#pragma unroll
    for (int k = 0; k < 3; ++k)
      for (int w = 0; w < 8; ++w) run[k] += wtot[w][k];
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_draft(const Geom& g, const Layout& L, void* ws, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(at<char>(ws, L, R_HIST), 0, L.size[R_HIST], st);
  if (e != cudaSuccess) return e;
  const int t = (g.nb + kLT - 1) / kLT;
  draft_logits_kernel<<<dim3(t, t, g.BH), 256, 0, st>>>(
      g, at<float>(ws, L, R_Q_AVG), at<float>(ws, L, R_K_AVG), at<float>(ws, L, R_Q_MAX),
      at<float>(ws, L, R_K_MAX), at<float>(ws, L, R_SCORES), at<float>(ws, L, R_LOGB));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  draft_mix_kernel<<<dim3(g.nb, g.BH), 256, 0, st>>>(g, at<float>(ws, L, R_SCORES),
                                                     at<float>(ws, L, R_LOGB),
                                                     at<unsigned int>(ws, L, R_HIST));
  return cudaGetLastError();
}

cudaError_t launch_rank(const Geom& g, const Layout& L, void* ws, bool hist0_done,
                        cudaStream_t st) {
  cudaError_t e;
  float* scores = at<float>(ws, L, R_SCORES);
  unsigned int* hist = at<unsigned int>(ws, L, R_HIST);
  RankState* rs = at<RankState>(ws, L, R_RSTATE);
  const long long P = (long long)g.nb * g.nb;
  const int per_cta = 16384;
  const int nchunk = (int)((P + per_cta - 1) / per_cta);
  if (!hist0_done) {
    if ((e = cudaMemsetAsync(hist, 0, L.size[R_HIST], st)) != cudaSuccess) return e;
  }
  rank_init_kernel<<<g.BH, 32, 0, st>>>(g, rs);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int pass = 0; pass < kRankPasses; ++pass) {
    const bool shared0 = pass == 0;
    if (pass > 0 || !hist0_done) {
      // pass 0 counts every key once into target 0's histogram (shared by all cuts)
      rank_hist_kernel<<<dim3(nchunk, g.BH), 256, 0, st>>>(g, scores, rs, hist, pass, per_cta);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    rank_select_kernel<<<g.BH, 32, 0, st>>>(g, rs, hist, pass, shared0 ? 1 : 0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  rank_assign_kernel<<<dim3(g.nb, g.BH), 256, 0, st>>>(g, scores, rs, at<uint8_t>(ws, L, R_MAP),
                                                       at<uint16_t>(ws, L, R_LISTS),
                                                       at<int>(ws, L, R_COUNTS));
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free ranking (da2_rank_noalloc).
//
// Same kernels and launch order as launch_rank on caller-given scores, but the
// radix-select scratch (per-pass histograms and per-cut state) lives in this
// file-scope device array instead of a caller workspace, so the call needs no
// device allocation by anyone.  Every GPU that loads the library holds the
// array (DA2_NOALLOC_MAX_HEADS heads' worth, about 1.5 MB) until the process
// exits.  All calls on a device share it, so calls that overlap on the GPU
// race; the histograms are cleared at the start of every call and the state is
// rewritten by rank_init_kernel, so a call never depends on the previous one.
constexpr size_t kNoallocHistBytes =
    (size_t)kRankPasses * DA2_NOALLOC_MAX_HEADS * kTargets * 256 * sizeof(unsigned int);
constexpr size_t kNoallocBytes =
    kNoallocHistBytes + (size_t)DA2_NOALLOC_MAX_HEADS * kTargets * sizeof(RankState);
static __device__ __align__(256) unsigned char g_rank_scratch[kNoallocBytes];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_addr[64];                // device address of g_rank_scratch, per device ordinal
unsigned long long g_scratch_ctx[64];    // id of the context that address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context (0 if unknown).  A
// context created after cudaDeviceReset gets a new id, so an address cached
// for the old context is never reused.
unsigned long long current_ctx_id() {
  static std::once_flag once;
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// In host code `g_rank_scratch` names a host-side shadow, not device memory:
// the device address has to be looked up, with the device current, before a
// kernel can be given it.  That happens once per device and context (the
// first call on a device, and the first call after its context was reset).
cudaError_t rank_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long id = current_ctx_id();
  if (!g_scratch_addr[dev] || id == 0 || id != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_rank_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_ctx_id();  // the lookup made the context current
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}
}  // namespace

cudaError_t launch_rank_noalloc(const Geom& g, const float* scores, uint8_t* map, uint16_t* lists,
                                int* counts, cudaStream_t st) {
  if (g.BH > DA2_NOALLOC_MAX_HEADS) return cudaErrorInvalidValue;
  void* base = nullptr;
  cudaError_t e = rank_scratch_address(&base);
  if (e != cudaSuccess) return e;
  unsigned int* hist = static_cast<unsigned int*>(base);
  RankState* rs = reinterpret_cast<RankState*>(static_cast<char*>(base) + kNoallocHistBytes);
  const size_t used_hist = (size_t)kRankPasses * g.BH * kTargets * 256 * sizeof(unsigned int);
  if ((e = cudaMemsetAsync(hist, 0, used_hist, st)) != cudaSuccess) return e;
  const long long P = (long long)g.nb * g.nb;
  const int per_cta = 16384;
  const int nchunk = (int)((P + per_cta - 1) / per_cta);
  rank_init_kernel<<<g.BH, 32, 0, st>>>(g, rs);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int pass = 0; pass < kRankPasses; ++pass) {
    rank_hist_kernel<<<dim3(nchunk, g.BH), 256, 0, st>>>(g, scores, rs, hist, pass, per_cta);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    rank_select_kernel<<<g.BH, 32, 0, st>>>(g, rs, hist, pass, pass == 0 ? 1 : 0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  rank_assign_kernel<<<dim3(g.nb, g.BH), 256, 0, st>>>(g, scores, rs, map, lists, counts);
  return cudaGetLastError();
}

}  // namespace da2
