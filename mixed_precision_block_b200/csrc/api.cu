// C-ABI entry points of libda2.so: argument validation, geometry, workspace
// layout, and the launch sequence of each stage.  See include/da2.h.
#include <cmath>
#include <cstring>

#include "da2_internal.cuh"

using namespace da2;

namespace {

int permille(float pct) { return (int)std::lrint(10.0 * (double)pct); }

int check_device() {
  static int cached[64];  // 0 = unknown, 1 = ok, 2 = unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DA2_ERR_CUDA;
  if (dev < 0 || dev >= 64) return DA2_ERR_UNSUPPORTED;
  if (cached[dev] == 0) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return DA2_ERR_CUDA;
    cached[dev] = (major == 10) ? 1 : 2;
  }
  return cached[dev] == 1 ? DA2_OK : DA2_ERR_UNSUPPORTED;
}

int make_geom(const da2_problem* p, Geom* g) {
  if (!p || !g) return DA2_ERR_ARG;
  if (p->B <= 0 || p->H <= 0 || p->T <= 0 || p->Hh <= 0 || p->Ww <= 0) return DA2_ERR_ARG;
  if (p->rh <= 0 || p->rw <= 0) return DA2_ERR_ARG;
  if (p->d != 64 && p->d != 128) return DA2_ERR_UNSUPPORTED;
  if (p->rh * p->rw != kBlockTokens) return DA2_ERR_UNSUPPORTED;
  if (!(p->lambda >= 0.f && p->lambda <= 1.f)) return DA2_ERR_ARG;
  double sum = 0;
  for (int i = 0; i < 4; ++i) {
    if (!(p->budget_pct[i] >= 0.f) || !(p->budget_pct[i] <= 100.f)) return DA2_ERR_ARG;
    sum += p->budget_pct[i];
  }
  if (std::fabs(sum - 100.0) > 0.2) return DA2_ERR_ARG;
  const int q4 = permille(p->budget_pct[1]), q8 = permille(p->budget_pct[2]),
            q16 = permille(p->budget_pct[3]);
  if (q4 + q8 + q16 > 1000) return DA2_ERR_ARG;
  g->B = p->B; g->H = p->H; g->T = p->T; g->Hh = p->Hh; g->Ww = p->Ww; g->d = p->d;
  g->rh = p->rh; g->rw = p->rw;
  g->nry = (p->Hh + p->rh - 1) / p->rh;
  g->nrx = (p->Ww + p->rw - 1) / p->rw;
  const long long nb = (long long)p->T * g->nry * g->nrx;
  const long long N = (long long)p->T * p->Hh * p->Ww;
  if (nb > 65535 || N > (1LL << 30) || (long long)p->B * p->H > (1LL << 20)) return DA2_ERR_UNSUPPORTED;
  g->nb = (int)nb;
  g->N = (int)N;
  g->BH = p->B * p->H;
  g->lambda = p->lambda;
  const long long P = nb * nb;
  auto cnt = [&](int cum) { return (P * cum + 500) / 1000; };
  const long long c16 = cnt(q16), c8 = cnt(q16 + q8), c4 = cnt(q16 + q8 + q4);
  g->n16 = c16; g->n8 = c8 - c16; g->n4 = c4 - c8;
  g->cut[0] = c16; g->cut[1] = c8; g->cut[2] = c4;
  return DA2_OK;
}

int check_ws(const Layout& L, const void* ws, size_t ws_bytes) {
  if (!ws || ((uintptr_t)ws & 255) != 0) return DA2_ERR_WORKSPACE;
  if (ws_bytes < L.total) return DA2_ERR_WORKSPACE;
  return DA2_OK;
}

bool aligned16(const void* p) { return p && ((uintptr_t)p & 15) == 0; }

// cudaErrorNotSupported is what the launchers return for a problem or driver
// the kernels do not cover (no fallback kernel exists).
int cuda_status(cudaError_t e) {
  return e == cudaSuccess ? DA2_OK : (e == cudaErrorNotSupported ? DA2_ERR_UNSUPPORTED : DA2_ERR_CUDA);
}

// Host-buffer path: the (batch, head) slices run in chunks of G, each chunk a
// problem of its own (B = 1, H = chunk size; every stage is per head).  Two
// sets of device buffers alternate so that one chunk's copies overlap the
// other's kernels.
struct HostPlan {
  da2_problem pc;   // chunk problem, H = G
  int BH, G, nchunks;
  size_t slice;     // bytes of one (b, h) slice of Q, K, V or O (bf16)
  size_t chunk;     // bytes of one chunk of one tensor, 256-aligned
  size_t ws;        // workspace bytes of a full chunk
  size_t set;       // q, k, v, out and workspace of one set
  size_t status;    // per-chunk status words after the two sets
  size_t status_off;  // the status word's offset in a chunk workspace
};

int host_plan(const da2_problem* p, int heads_per_chunk, HostPlan* hp) {
  Geom g;
  int rc = make_geom(p, &g);
  if (rc) return rc;
  if (heads_per_chunk <= 0) return DA2_ERR_ARG;
  hp->BH = g.BH;
  hp->G = heads_per_chunk < g.BH ? heads_per_chunk : g.BH;
  hp->nchunks = (g.BH + hp->G - 1) / hp->G;
  hp->pc = *p;
  hp->pc.B = 1;
  hp->pc.H = hp->G;
  Geom gc;
  if ((rc = make_geom(&hp->pc, &gc))) return rc;
  hp->slice = (size_t)g.N * g.d * 2;
  hp->chunk = (hp->slice * hp->G + 255) & ~(size_t)255;
  const Layout Lc = make_layout(gc);
  hp->ws = Lc.total;
  hp->status_off = Lc.off[R_STATUS];
  hp->set = 4 * hp->chunk + hp->ws;
  hp->status = ((size_t)hp->nchunks * 2 * sizeof(int) + 255) & ~(size_t)255;  // two status words per chunk
  return DA2_OK;
}

}  // namespace

extern "C" {

int da2_plan(const da2_problem* p, da2_plan_info* out) {
  Geom g;
  int rc = make_geom(p, &g);
  if (rc) return rc;
  if (!out) return DA2_ERR_ARG;
  const Layout L = make_layout(g);
  out->pairs_per_head = (long long)g.nb * g.nb;
  out->n16 = g.n16; out->n8 = g.n8; out->n4 = g.n4;
  out->nskip = out->pairs_per_head - g.cut[2];
  out->nb = g.nb; out->nry = g.nry; out->nrx = g.nrx; out->N = g.N;
  out->Np = g.nb * kBlockTokens;
  out->ws_bytes = L.total;
  return DA2_OK;
}

int da2_prepare(const da2_problem* p, const void* q, const void* k, const void* v,
                void* ws, size_t ws_bytes, void* stream) {
  Geom g;
  int rc = make_geom(p, &g);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return DA2_ERR_ARG;
  const Layout L = make_layout(g);
  if ((rc = check_ws(L, ws, ws_bytes))) return rc;
  if ((rc = check_device())) return rc;
  return cuda_status(launch_prepare(g, L, q, k, v, ws, (cudaStream_t)stream));
}

int da2_draft_rank(const da2_problem* p, void* ws, size_t ws_bytes, void* stream) {
  Geom g;
  int rc = make_geom(p, &g);
  if (rc) return rc;
  const Layout L = make_layout(g);
  if ((rc = check_ws(L, ws, ws_bytes))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = launch_draft(g, L, ws, st);
  if (e == cudaSuccess) e = launch_rank(g, L, ws, /*hist0_done=*/true, st);
  // the attention kernel walks query blocks in pairs: their merged key lists
  if (e == cudaSuccess) e = launch_pair_lists(g, L, ws, st);
  return cuda_status(e);
}

int da2_rank_from_scores(const da2_problem* p, const float* scores, void* ws,
                         size_t ws_bytes, void* stream) {
  Geom g;
  int rc = make_geom(p, &g);
  if (rc) return rc;
  if (!aligned16(scores)) return DA2_ERR_ARG;
  const Layout L = make_layout(g);
  if ((rc = check_ws(L, ws, ws_bytes))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(at<float>(ws, L, R_SCORES), scores, L.size[R_SCORES],
                                  cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = launch_rank(g, L, ws, /*hist0_done=*/false, st);
  if (e == cudaSuccess) e = launch_pair_lists(g, L, ws, st);
  return cuda_status(e);
}

int da2_attention(const da2_problem* p, const void* q, const void* k, const void* v,
                  void* ws, size_t ws_bytes, void* out, void* stream) {
  Geom g;
  int rc = make_geom(p, &g);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DA2_ERR_ARG;
  const Layout L = make_layout(g);
  if ((rc = check_ws(L, ws, ws_bytes))) return rc;
  if ((rc = check_device())) return rc;
  return cuda_status(launch_attention(g, L, q, k, v, ws, out, (cudaStream_t)stream));
}

int da2_dense_attention(int B, int H, int N, int d, const void* q, const void* k,
                        const void* v, void* out, void* stream) {
  if (B <= 0 || H <= 0 || N <= 0) return DA2_ERR_ARG;
  if ((d != 64 && d != 128) || N < 64) return DA2_ERR_UNSUPPORTED;
  if ((long long)B * H > (1LL << 20) || N > (1 << 30)) return DA2_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DA2_ERR_ARG;
  int rc = check_device();
  if (rc) return rc;
  return cuda_status(launch_dense(B, H, N, d, q, k, v, out, (cudaStream_t)stream));
}

int da2_dense_check_status(void* stream) {
  int rc = check_device();
  if (rc) return rc;
  int word = 0;
  if (dense_status(&word, (cudaStream_t)stream) != cudaSuccess) return DA2_ERR_CUDA;
  return word ? DA2_ERR_TIMEOUT : DA2_OK;
}

int da2_attention_wait_test(const da2_problem* p, const void* q, const void* k, const void* v,
                            void* ws, size_t ws_bytes, void* out, int withheld_cta,
                            unsigned int wait_polls, void* stream) {
  Geom g;
  int rc = make_geom(p, &g);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || wait_polls == 0) return DA2_ERR_ARG;
  const Layout L = make_layout(g);
  if ((rc = check_ws(L, ws, ws_bytes))) return rc;
  if ((rc = check_device())) return rc;
  return cuda_status(launch_attention_test(g, L, q, k, v, ws, out, (cudaStream_t)stream, wait_polls,
                                           withheld_cta));
}

int da2_attention_occupancy(int d, int dense, int* ctas_per_sm) {
  if ((d != 64 && d != 128) || !ctas_per_sm) return DA2_ERR_ARG;
  int rc = check_device();
  if (rc) return rc;
  return cuda_status(attention_occupancy(d, dense != 0, ctas_per_sm));
}

int da2_debug_view(const da2_problem* p, void* ws, int which, void** ptr, size_t* bytes) {
  Geom g;
  int rc = make_geom(p, &g);
  if (rc) return rc;
  if (!ws || !ptr || !bytes) return DA2_ERR_ARG;
  static const Region map[DA2_VIEW_COUNT_] = {
      R_PERM, R_Q_AVG, R_K_AVG, R_Q_MAX, R_K_MAX, R_Q_I8, R_K_I8, R_Q_S8, R_K_S8,
      R_Q_F4, R_K_F4, R_Q_SF4, R_K_SF4, R_V_I8, R_V_S8, R_V_F4, R_V_SF4, R_V_G4,
      R_SCORES, R_MAP, R_LISTS, R_COUNTS, R_STATUS};
  if (which < 0 || which >= DA2_VIEW_COUNT_) return DA2_ERR_ARG;
  const Layout L = make_layout(g);
  *ptr = static_cast<char*>(ws) + L.off[map[which]];
  *bytes = L.size[map[which]];
  return DA2_OK;
}

int da2_rank_noalloc(const da2_problem* p, const float* scores, uint8_t* map, uint16_t* lists,
                     int32_t* counts, void* stream) {
  Geom g;
  int rc = make_geom(p, &g);
  if (rc) return rc;
  if (g.BH > DA2_NOALLOC_MAX_HEADS) return DA2_ERR_UNSUPPORTED;
  if (!aligned16(scores) || !aligned16(map) || !aligned16(lists) || !aligned16(counts)) return DA2_ERR_ARG;
  if ((rc = check_device())) return rc;
  return cuda_status(launch_rank_noalloc(g, scores, map, lists, counts, (cudaStream_t)stream));
}

int da2_check_status(const da2_problem* p, const void* ws, size_t ws_bytes, void* stream) {
  Geom g;
  int rc = make_geom(p, &g);
  if (rc) return rc;
  const Layout L = make_layout(g);
  if (!ws || ws_bytes < L.total) return DA2_ERR_WORKSPACE;
  // word 0: the attention kernel's, word 1: the preparation's
  int word[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(word, static_cast<const char*>(ws) + L.off[R_STATUS], sizeof(word),
                                  cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  return (word[0] | word[1]) ? DA2_ERR_TIMEOUT : DA2_OK;
}

int da2_host_bytes(const da2_problem* p, int heads_per_chunk, size_t* bytes) {
  HostPlan hp;
  int rc = host_plan(p, heads_per_chunk, &hp);
  if (rc) return rc;
  if (!bytes) return DA2_ERR_ARG;
  *bytes = 2 * hp.set + hp.status;
  return DA2_OK;
}

int da2_forward_host(const da2_problem* p, const void* q, const void* k, const void* v, void* out,
                     void* dev, size_t dev_bytes, int heads_per_chunk, void* stream) {
  HostPlan hp;
  int rc = host_plan(p, heads_per_chunk, &hp);
  if (rc) return rc;
  if (!q || !k || !v || !out) return DA2_ERR_ARG;
  if (!dev || ((uintptr_t)dev & 255) != 0 || dev_bytes < 2 * hp.set + hp.status) return DA2_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;
  cudaStream_t cs = (cudaStream_t)stream, hs = nullptr, ds = nullptr;
  cudaEvent_t start = nullptr, ev[3][2] = {};  // [copies in, kernels, copy out][set]
  cudaError_t e = cudaStreamCreateWithFlags(&hs, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&ds, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming);
  for (int i = 0; i < 3; ++i)
    for (int s = 0; s < 2; ++s)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev[i][s], cudaEventDisableTiming);
  // the copy streams start after whatever the caller queued on its stream
  if (e == cudaSuccess) e = cudaEventRecord(start, cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hs, start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ds, start, 0);
  int* status = reinterpret_cast<int*>(static_cast<char*>(dev) + 2 * hp.set);
  if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, hp.status, cs);
  for (int c = 0; c < hp.nchunks && e == cudaSuccess && rc == DA2_OK; ++c) {
    const int s = c & 1, h0 = c * hp.G, gh = (hp.BH - h0) < hp.G ? (hp.BH - h0) : hp.G;
    char* base = static_cast<char*>(dev) + s * hp.set;
    char *dq = base, *dk = base + hp.chunk, *dv = base + 2 * hp.chunk, *dout = base + 3 * hp.chunk;
    char* ws = base + 4 * hp.chunk;
    const size_t off = (size_t)h0 * hp.slice, nbytes = (size_t)gh * hp.slice;
    // copies in, once the kernels of the chunk two back released this set
    if (c >= 2) e = cudaStreamWaitEvent(hs, ev[1][s], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dq, static_cast<const char*>(q) + off, nbytes, cudaMemcpyHostToDevice, hs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dk, static_cast<const char*>(k) + off, nbytes, cudaMemcpyHostToDevice, hs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dv, static_cast<const char*>(v) + off, nbytes, cudaMemcpyHostToDevice, hs);
    if (e == cudaSuccess) e = cudaEventRecord(ev[0][s], hs);
    // the kernels, once the copies are in and the output of the chunk two back is out
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev[0][s], 0);
    if (e == cudaSuccess && c >= 2) e = cudaStreamWaitEvent(cs, ev[2][s], 0);
    if (e != cudaSuccess) break;
    da2_problem pcc = hp.pc;
    pcc.H = gh;
    if ((rc = da2_prepare(&pcc, dq, dk, dv, ws, hp.ws, cs)) == DA2_OK &&
        (rc = da2_draft_rank(&pcc, ws, hp.ws, cs)) == DA2_OK)
      rc = da2_attention(&pcc, dq, dk, dv, ws, hp.ws, dout, cs);
    if (rc != DA2_OK) break;
    // the chunk's bounded-wait status words (the next use of the workspace clears them)
    e = cudaMemcpyAsync(status + 2 * c, ws + hp.status_off, 2 * sizeof(int), cudaMemcpyDeviceToDevice, cs);
    if (e == cudaSuccess) e = cudaEventRecord(ev[1][s], cs);
    // copy out
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ds, ev[1][s], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(static_cast<char*>(out) + off, dout, nbytes, cudaMemcpyDeviceToHost, ds);
    if (e == cudaSuccess) e = cudaEventRecord(ev[2][s], ds);
  }
  // the call returns with the output on the host
  const cudaError_t e1 = cudaStreamSynchronize(hs), e2 = cudaStreamSynchronize(cs), e3 = cudaStreamSynchronize(ds);
  if (e == cudaSuccess) e = e1 != cudaSuccess ? e1 : (e2 != cudaSuccess ? e2 : e3);
  if (e == cudaSuccess && rc == DA2_OK) {
    for (int c = 0; c < hp.nchunks && e == cudaSuccess; ++c) {
      int word[2] = {0, 0};
      e = cudaMemcpy(word, status + 2 * c, sizeof(word), cudaMemcpyDeviceToHost);
      if (word[0] | word[1]) rc = DA2_ERR_TIMEOUT;
    }
  }
  for (int i = 0; i < 3; ++i)
    for (int s = 0; s < 2; ++s)
      if (ev[i][s]) cudaEventDestroy(ev[i][s]);
  if (start) cudaEventDestroy(start);
  if (hs) cudaStreamDestroy(hs);
  if (ds) cudaStreamDestroy(ds);
  if (rc != DA2_OK) return rc;
  return cuda_status(e);
}

const char* da2_status_string(int s) {
  switch (s) {
    case DA2_OK: return "ok";
    case DA2_ERR_ARG: return "invalid argument";
    case DA2_ERR_UNSUPPORTED: return "unsupported problem or device";
    case DA2_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DA2_ERR_CUDA: return "CUDA launch or runtime error";
    case DA2_ERR_TIMEOUT: return "a bounded wait in an attention kernel expired";
    default: return "unknown status";
  }
}

}  // extern "C"
