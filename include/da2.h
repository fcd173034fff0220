/*
 * da2.h — C ABI of libda2.so, a B200 (sm_100a) implementation of the
 * DraftAttention2 low-resolution-guided mixed-precision block-sparse attention.
 *
 * Sources, cited by page title and section:
 *   [abstract]  DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided
 *               Mixed-Precision Attention — Abstract.
 *   [note]      DraftAttention2 reading note (Chinese blog post on the same
 *               paper) — "Method overview" bullets 1-4, Figure 2 and Figure 3
 *               captions, experiment section.
 *   [v1]        DraftAttention: Fast Video Diffusion via Low-Resolution
 *               Attention Guidance — Abstract.
 *
 * One attention call is three entry points enqueued on one stream:
 *   da2_prepare     reorder Q/K/V into region blocks, pool, quantise
 *   da2_draft_rank  draft map, shared per-head ranking, precision assignment
 *   da2_attention   mixed-precision attention, output restored to token order
 *
 * Conventions (all entry points):
 *   - Q, K, V and the output are bf16, contiguous [B, H, N, d] with
 *     N = T*Hh*Ww and token n = (t*Hh + y)*Ww + x; device pointers, 16-byte
 *     aligned.  The caller owns every buffer.
 *   - `ws` is a caller-allocated device workspace of at least
 *     da2_plan_info.ws_bytes bytes (256-byte aligned); it carries the prepared
 *     operands and the assignment from one call to the next, so the three calls
 *     of one attention must use the same workspace and problem.  The library
 *     allocates no device memory and keeps no state between calls beyond
 *     per-device function attributes; calls with distinct workspaces may run
 *     concurrently on different streams.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All device work is asynchronous on that stream.
 *   - Return value: DA2_OK or an error code; nothing throws across the ABI.
 *     Argument errors are detected on the host before any launch.  A launch
 *     failure returns DA2_ERR_CUDA.
 */
#ifndef DA2_H
#define DA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  DA2_OK = 0,
  DA2_ERR_ARG = 1,          /* invalid sizes, pointers, lambda or budget       */
  DA2_ERR_UNSUPPORTED = 2,  /* d not in {64,128}, rh*rw != 64, no sm_100 GPU,
                               no TMA tensor-map encoder in the driver          */
  DA2_ERR_WORKSPACE = 3,    /* workspace NULL, misaligned or too small         */
  DA2_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed            */
  DA2_ERR_TIMEOUT = 5       /* a device-side bounded wait expired (see below)  */
};

/* Problem statement of one attention call.
 * Region size rh x rw cuts every frame's Hh x Ww grid into regions; frames are
 * padded to multiples of the region size and padding tokens are masked
 * ([note] Figure 3(a)).  rh*rw must be 64 (one region = one 64-token block).
 * lambda in [0,1] weights the max-pooled draft map ([note] Method overview
 * bullet 1; lambda = 0 is average-only drafting, [v1]).
 * budget_pct = {skip, 4-bit, 8-bit, 16-bit} percentages of the region pairs of
 * each head ([note] experiment section, "Bit" column 0/4/8/16).  The 4/8/16
 * shares must be >= 0 with sum <= 100; the four must sum to 100 within 0.2
 * (published budgets are rounded, e.g. 80.7/14.4/4.8/0); skip is taken as the
 * remainder. */
typedef struct da2_problem {
  int B, H, T, Hh, Ww, d;
  int rh, rw;
  float lambda;
  float budget_pct[4];
} da2_problem;

/* Derived sizes.  Counts are per (batch, head): with P = nb^2 pairs and
 * permille shares q = round(10*pct), cumulative counts c = floor((P*cum+500)/1000)
 * taken in order 16, 8, 4. */
typedef struct da2_plan_info {
  long long pairs_per_head;
  long long n16, n8, n4, nskip;
  int nb, nry, nrx, N, Np;
  size_t ws_bytes;
} da2_plan_info;

/* Validates `p` and fills `out`.  Host only, no device work. */
int da2_plan(const da2_problem* p, da2_plan_info* out);

/* Stage 1 ([abstract]; [note] Method overview bullet 4, Figure 3(b)).
 * Per (batch, head, region block): the block's 64 tokens are gathered from
 * Q and K, their average and channel-wise max descriptors are pooled over the
 * region's real tokens, and Q/K are quantised to INT8 (one fp32 scale per
 * block) and NVFP4 (e4m3 scale per 16 channels of a token).  V is quantised
 * per channel (INT8; NVFP4 with a per-channel fp32 scale and e4m3 scales per
 * 16 tokens) and transposed to [block][channel][token].  Formats the budget
 * does not use are not written.  q, k, v: device bf16 [B,H,N,d].  V crosses
 * HBM about once: one persistent kernel merges a head's channel absmax and
 * writes its codes one head later, from L2, after a bounded wait whose expiry
 * sets the second status word (da2_check_status). */
int da2_prepare(const da2_problem* p, const void* q, const void* k, const void* v,
                void* ws, size_t ws_bytes, void* stream);

/* Stage 2 ([abstract]; [note] Method overview bullets 1-2, Figure 2).
 * Draft map D = (1-lambda)*softmax(avgQ avgK^T/sqrt d) + lambda*softmax(maxQ maxK^T/sqrt d)
 * per head over region pairs (fp32), then one ranking per head, descending by D
 * with ties broken by ascending pair index q_block*nb + k_block, hands out the
 * budget: first n16 pairs 16-bit, next n8 INT8, next n4 NVFP4, rest skipped.
 * Also builds, per pair of neighbouring query blocks (2p, 2p+1), the merged
 * key lists the attention kernel walks.
 * Requires da2_prepare on the same workspace first. */
int da2_draft_rank(const da2_problem* p, void* ws, size_t ws_bytes, void* stream);

/* Test hook for stage 2: ranking, assignment and the pair lists only, on
 * caller-given fp32 scores [B,H,nb,nb] (device), which are copied into the
 * workspace first. */
int da2_rank_from_scores(const da2_problem* p, const float* scores, void* ws,
                         size_t ws_bytes, void* stream);

/* Stage 3 ([abstract]; [note] Method overview bullets 3-4; [v1] order restore).
 * Per query block one pass runs the 16-bit phase (bf16 Q/K/V), the INT8 phase
 * and the NVFP4 phase over its assigned key blocks with one shared online
 * softmax state and one fp32 output accumulator.  Low-bit P is quantised per
 * (query row, key block) against that block's own row maximum rounded up to
 * a power of two, r = ceil(max x) over the block's real keys (x = s log2 e):
 * INT8 codes round(255 * 2^(x - r)); NVFP4 of 2688 * 2^(x - r) per 16 keys.
 * Each low-bit block enters numerator and row sum with the same quantised
 * weights, and each phase joins the shared accumulator with its V channel
 * scale.  The output rows are written straight back to the
 * original token order (padding rows dropped); a query block with no key
 * block outputs zeros.
 * q, k, v: the same device tensors given to da2_prepare; out: device bf16
 * [B,H,N,d].  Requires da2_draft_rank (or da2_rank_from_scores) first.
 * Every wait inside the kernel is bounded: read the outcome with
 * da2_check_status.  Returns DA2_ERR_UNSUPPORTED when the driver lacks the
 * TMA tensor-map encoder the kernel needs (there is no other kernel). */
int da2_attention(const da2_problem* p, const void* q, const void* k, const void* v,
                  void* ws, size_t ws_bytes, void* out, void* stream);

/* Own dense bf16 softmax attention over all N tokens (the comparison point
 * for the sparse path): out = softmax(q k^T / sqrt d) v, fp32 accumulation,
 * bf16 output.  q, k, v, out: device bf16 [B,H,N,d]; d in {64,128}, N >= 64
 * (otherwise DA2_ERR_UNSUPPORTED).  It runs the sparse path's tensor-core
 * kernel with every key block in the 16-bit phase, over 64-token blocks in
 * natural order.  Needs no workspace; its bounded-wait status goes to a word
 * inside the library, read with da2_dense_check_status.  No counterpart on
 * the pages beyond dense attention itself. */
int da2_dense_attention(int B, int H, int N, int d, const void* q, const void* k,
                        const void* v, void* out, void* stream);

/* Status of the dense calls on the current device since the last
 * da2_dense_attention was enqueued: synchronises `stream`, returns DA2_OK, or
 * DA2_ERR_TIMEOUT if a bounded wait in a dense kernel expired (its output is
 * then incomplete), or DA2_ERR_CUDA.  Dense calls share the word, so
 * concurrent dense calls on one device report together. */
int da2_dense_check_status(void* stream);

/* Test hook for the failure path, no counterpart on the pages: runs
 * da2_attention with every bounded wait limited to `wait_polls` polls and
 * with CTA `withheld_cta` (blockIdx.x; -1 for none) never issuing its first
 * key-tile load, so that the waits on that tile run out.  The kernel then
 * raises the workspace status word, stops issuing work, waits (bounded) for
 * its copies in flight and releases its tensor memory; da2_check_status
 * returns DA2_ERR_TIMEOUT.  Nothing faults and the context stays usable. */
int da2_attention_wait_test(const da2_problem* p, const void* q, const void* k, const void* v,
                            void* ws, size_t ws_bytes, void* out, int withheld_cta,
                            unsigned int wait_polls, void* stream);

/* Introspection, no counterpart on the pages: *ctas_per_sm receives how many
 * CTAs of the attention kernel for head dimension d (64 or 128; dense != 0:
 * the dense kernel) one SM holds at once.  The kernel is laid out for 1 CTA
 * per SM (it allocates all 512 TMEM columns, 384 threads at 168 registers)
 * holding two query-block pairs, whose softmax warpgroups hide each other's
 * latency.  Sets the kernel's launch attributes as a call would; no device
 * work.  DA2_ERR_ARG for another d or a null pointer. */
int da2_attention_occupancy(int d, int dense, int* ctas_per_sm);

/* Workspace views for tests.  Returns the device address and size of one
 * intermediate inside `ws` (no device work).  Layouts (bh = b*H + h):
 *   PERM   int32 [nb][64]            token of each block slot, -1 = padding
 *   Q_AVG/K_AVG/Q_MAX/K_MAX  fp32 [B*H][nb][d]
 *   Q_I8/K_I8  int8 [B*H][nb][64][d];  Q_S8/K_S8 fp32 [B*H][nb]
 *   Q_F4/K_F4  uint8 [B*H][nb][64][d/2] (even channel in the low nibble)
 *   Q_SF4/K_SF4 uint8 e4m3 [B*H][nb][d/64][32][16]: per 64-channel chunk an
 *          atom whose line i holds the 4 scales (16 channels each) of slots i
 *          and i+32 as two 32-bit words, repeated in words 2-3 (the layout the
 *          tensor core reads scale factors from)
 *   V_I8  bf16 [B*H][nb][64][d]: V's INT8 codes (integers -127..127, exact
 *          as bf16) in block slot order, the operand layout of the P.V MMA;
 *          V_S8 fp32 [B*H][d]
 *   V_F4  uint8 [B*H][nb][d][32] (even token in the low nibble)
 *   V_SF4 uint8 e4m3 [B*H][nb][32][16]: line i holds the 4 scales (16 tokens
 *          each) of channels i, i+32, i+64, i+96;  V_G4 fp32 [B*H][d]
 *   SCORES fp32 [B*H][nb][nb]
 *   MAP    uint8 [B*H][nb][nb]  precision per pair: 16, 8, 4 or 0 (skip)
 *   LISTS  uint16 [B*H][nb][nb] per query block: its 16-bit key blocks, then
 *          its 8-bit, then its 4-bit ones, each ascending
 *   COUNTS int32 [B*H][nb][4]   lengths of the three lists, 0
 *   STATUS int32 [2]            word 0: 0, or 1 after a tensor-core attention
 *                               call whose bounded pipeline waits expired (its
 *                               output is then invalid), reset by every
 *                               da2_attention; word 1: the same for the V
 *                               preparation, reset by every da2_prepare */
enum {
  DA2_VIEW_PERM = 0,
  DA2_VIEW_Q_AVG, DA2_VIEW_K_AVG, DA2_VIEW_Q_MAX, DA2_VIEW_K_MAX,
  DA2_VIEW_Q_I8, DA2_VIEW_K_I8, DA2_VIEW_Q_S8, DA2_VIEW_K_S8,
  DA2_VIEW_Q_F4, DA2_VIEW_K_F4, DA2_VIEW_Q_SF4, DA2_VIEW_K_SF4,
  DA2_VIEW_V_I8, DA2_VIEW_V_S8, DA2_VIEW_V_F4, DA2_VIEW_V_SF4, DA2_VIEW_V_G4,
  DA2_VIEW_SCORES, DA2_VIEW_MAP, DA2_VIEW_LISTS, DA2_VIEW_COUNTS, DA2_VIEW_STATUS,
  DA2_VIEW_COUNT_
};
int da2_debug_view(const da2_problem* p, void* ws, int which, void** ptr, size_t* bytes);

/* Allocation-free ranking.  The paper has no counterpart: this entry point
 * exists for callers that cannot allocate device memory at call time — for
 * example a host runtime that hands every byte of the GPU to its own arena at
 * start-up, or a plugin hook invoked from another engine's execution path
 * where allocating is not permitted — and so cannot provide the workspace
 * that da2_rank_from_scores needs for its radix-select histograms.
 *
 * It computes exactly what da2_rank_from_scores computes (ranking and
 * precision assignment of caller-given fp32 scores [B,H,nb,nb]) and writes the
 * results to caller-given device buffers with the layouts of the MAP, LISTS
 * and COUNTS workspace views: map uint8 [B,H,nb,nb], lists uint16 [B,H,nb,nb]
 * (only the first c16+c8+c4 entries of a row are written), counts int32
 * [B,H,nb,4].  All pointers are device pointers, 16-byte aligned.
 *
 * Scratch: a fixed array inside the library, sized for at most
 * DA2_NOALLOC_MAX_HEADS (batch x head) pairs; larger problems return
 * DA2_ERR_UNSUPPORTED before any device work.  Every GPU that loads the
 * library keeps that array (about 1.5 MB) until the process exits.  The first
 * call on a device (and the first after that device's context was reset)
 * looks the array's device address up (a runtime call) and keeps it for that
 * context; make that first call before any stream capture.  Calls on one device share the
 * array: calls that may overlap on the GPU (different streams, no ordering)
 * race and give wrong results; serialise them.  No call depends on what an
 * earlier call left in the array.  The call allocates nothing: no cudaMalloc,
 * no cudaFree, no allocating library routine. */
#define DA2_NOALLOC_MAX_HEADS 64
int da2_rank_noalloc(const da2_problem* p, const float* scores, uint8_t* map, uint16_t* lists,
                     int32_t* counts, void* stream);

/* Device status of the last da2_prepare and da2_attention on `ws`: synchronises
 * `stream`, reads the workspace's two status words and returns DA2_OK, or
 * DA2_ERR_TIMEOUT if a bounded wait inside the V preparation or the attention
 * kernel expired (the output is then incomplete), or DA2_ERR_CUDA if the
 * stream reports an error.  No counterpart on the pages: it reports this
 * implementation's own wait bounds. */
int da2_check_status(const da2_problem* p, const void* ws, size_t ws_bytes, void* stream);

/* Host-buffer form of the whole path (da2_prepare, da2_draft_rank and
 * da2_attention) for callers whose Q/K/V and output live in host memory.
 * The (batch, head) slices run in chunks of heads_per_chunk, each chunk a
 * problem of its own (every stage is per head: DraftAttention2 reading note,
 * Method overview bullets 1-4, one ranking per head); two sets of device
 * buffers alternate so that the host<->device copies of one chunk overlap the
 * kernels of another.  No counterpart on the pages.
 *
 * da2_host_bytes: bytes of the device buffer da2_forward_host needs for this
 * problem and chunk size (two sets of chunk Q, K, V, output and workspace,
 * plus one status word per chunk).
 *
 * da2_forward_host: q, k, v: host [B,H,T*Hh*Ww,d] bf16, read; out: host
 * [B,H,N,d] bf16, written in token order.  Host buffers should be page-locked
 * (cudaHostAlloc / cudaHostRegister) for the copies to run asynchronously;
 * pageable memory is correct but serialises them.  dev: caller-owned device
 * buffer of at least da2_host_bytes bytes, 256-byte aligned.  stream: work
 * already queued on it runs first; the call creates two copy streams of its
 * own for its duration.  Synchronous: returns once the output is on the host.
 * Returns DA2_OK, DA2_ERR_ARG / _UNSUPPORTED (problem, as da2_plan),
 * DA2_ERR_WORKSPACE (dev missing, misaligned or too small), DA2_ERR_TIMEOUT
 * (a bounded wait in some chunk's attention kernel expired) or DA2_ERR_CUDA. */
int da2_host_bytes(const da2_problem* p, int heads_per_chunk, size_t* bytes);
int da2_forward_host(const da2_problem* p, const void* q, const void* k, const void* v, void* out,
                     void* dev, size_t dev_bytes, int heads_per_chunk, void* stream);

/* Human-readable name of a status code (static string). */
const char* da2_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* DA2_H */
