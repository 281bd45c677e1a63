/*
 * pa.h -- C ABI of libpa: partition attention with attention-state merge, selective
 * reuse and partition importance on one NVIDIA B200 (sm_100a).
 *
 * What the calls compute (web summaries of DiTango, "Cost-Effective Parallel Diffusion
 * Generation with Selective Attention State Reuse", and SwiftFusion, "Scalable Sequence
 * Parallelism for Distributed Inference of Diffusion Transformers on GPUs"):
 *
 *   pa_partition_attn    the attention state (partial output O_p, log-sum-exp LSE_p) of
 *                        each query row against one KV partition, for the (query group,
 *                        KV group) pairs selected as fresh -- DiTango, Methodology 2,
 *                        "State Composition" (states of output and log-sum-exp) and
 *                        "Group-wise state computation".
 *   pa_merge_states      the associative, commutative composition of those states,
 *                        taking per (query group, KV group) either the fresh state or the
 *                        cached state of an earlier step -- DiTango, Methodology 1
 *                        ("Anchor-Guided Selection Planner": recompute or reuse) and
 *                        Methodology 2 ("State Composition").
 *   pa_importance        partition importance w_p = exp(LSE_p - LSE), averaged per
 *                        (query group, partition) -- DiTango, Methodology 1 ("Error
 *                        modelling", "Anchor steps": importance refreshed at anchors).
 *   pa_state_drift       per (query group, partition) sums of the squared change of the
 *                        states between two steps and of the reference states' squares:
 *                        the measurement behind the online prediction between anchor
 *                        steps -- DiTango, Methodology 1 ("Online Prediction": the change
 *                        of the always-computed local states stands in for the drift of
 *                        the reused remote ones).
 *   pa_relayout_seq2head the sequence-major -> head-major permutation that the Ulysses
 *                        all-to-all performs, in sequence chunks -- SwiftFusion,
 *                        Methodology 2 ("Torus Attention": the all-to-all split into
 *                        chunks that overlap compute).
 *
 * Notation.  B batch, H heads, N tokens, D head dim (64 or 128).  P partitions (1..128)
 * given by part_off[0..P] (part_off[0] = 0, non-decreasing, part_off[P] = N); partition p
 * covers tokens [part_off[p], part_off[p+1]).  A group is G consecutive partitions, for
 * queries and keys alike: QG = KG = ceil(P / G); query group g covers tokens
 * [part_off[g*G], part_off[min((g+1)*G, P)]).  fresh[qg*KG + kg] != 0 selects the pair
 * (query group qg, KV group kg) for fresh computation.
 *
 * Math.  For query row i and partition p with valid keys J_p:
 *   s_ij = scale * <q_i, k_j>,  LSE_p(i) = ln sum_{j in J_p} exp(s_ij),
 *   O_p(i) = sum_{j in J_p} exp(s_ij - LSE_p(i)) v_j,
 *   LSE(i) = ln sum_p exp(LSE_p(i)),  O(i) = sum_p exp(LSE_p(i) - LSE(i)) O_p(i),
 *   w[qg][p] = mean over b, h and rows i of qg of exp(LSE_p(i) - LSE(i)).
 * An empty partition has LSE_p = -inf and O_p = 0.
 *
 * Layouts (row-major, contiguous, all device memory unless marked host):
 *   q, k, v        [B][H][N][D]            dtype (head-major)
 *   o_part         [P][B][H][N][D]         dtype
 *   lse_part       [P][B][H][N]            float32, natural log
 *   o              [B][H][N][D]            dtype
 *   lse            [B][H][N]               float32
 *   w              [QG][P]                 float32
 *   relayout src   [N][H][D], dst [H][N][D], elem_bytes each
 *
 * Ownership.  The caller allocates and owns every buffer; the library never frees or
 * retains caller memory past the call.  A pa_ctx owns only its own device workspace and
 * an error-status word.  Calls are asynchronous on the given stream (a cudaStream_t
 * passed as void*; NULL = the legacy default stream): they validate, enqueue kernels
 * and return.  No call synchronises except pa_sync_status, and a call that first needs a
 * larger workspace (cudaFree of the old one and cudaMalloc synchronise the device).  The
 * calls that use the workspace -- pa_merge_states with w, pa_importance, pa_state_drift
 * -- share it, so on one context they must not overlap on the GPU (issue them on one
 * stream, or use a context per stream).
 *
 * Debug.  With PA_DEBUG set (not "0") in the environment when pa_init runs, every call on
 * that context synchronises its stream after launching and returns what pa_sync_status
 * would (PA_ECUDA for a launch or runtime error, PA_ETIMEOUT for a device-side wait that
 * gave up).
 *
 * Fault injection (tests).  PA_INJECT_ENOMEM, a comma-separated list of the sites "init"
 * (pa_init's status word) and "workspace" (the context workspace), read at each device
 * allocation, makes those allocations fail with PA_ENOMEM as if cudaMalloc had, without
 * calling it; the call then behaves as under real memory pressure (pa_init returns no
 * context; a workspace call returns PA_ENOMEM, launches nothing and leaves the context
 * usable).
 *
 * Errors.  Every call returns PA_OK (0) or a negative status; pa_last_error gives a
 * one-line message for the last failure on that context (thread-unsafe per context).
 * Validation happens before anything is enqueued: on error nothing was launched.
 * Device-side waits are bounded; a wait that gives up records PA_ETIMEOUT in the
 * context's status word, which pa_sync_status reads (and clears).
 *
 * Alignment.  q, k, v, o_part, o and relayout src/dst must be 16-byte aligned;
 * lse_part, lse, w 4-byte aligned.
 */
#ifndef PA_H
#define PA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_MAX_P 128

enum {
  PA_OK = 0,
  PA_EINVAL = -1,        /* bad argument (null pointer, size, offsets, mask) */
  PA_EALIGN = -2,        /* pointer misaligned */
  PA_EUNSUPPORTED = -3,  /* device is not sm_100, or dtype / D not supported */
  PA_ENOMEM = -4,        /* workspace allocation failed */
  PA_ECUDA = -5,         /* a CUDA runtime call or launch failed */
  PA_ETIMEOUT = -6       /* a device-side wait gave up (reported by pa_sync_status) */
};

typedef enum { PA_F32 = 0, PA_BF16 = 1 } pa_dtype;

typedef struct pa_ctx pa_ctx;

/* Create a context on CUDA device `device`.  Rejects devices other than compute
 * capability 10.0 (PA_EUNSUPPORTED).  On success *out owns a small device status word.
 * On failure *out is NULL and pa_last_error(NULL) gives the reason. */
int pa_init(int device, pa_ctx** out);

/* Release a context and its device memory.  NULL is a no-op.  The caller must ensure no
 * call on this context is still executing on the GPU. */
void pa_destroy(pa_ctx* ctx);

/* Message of the last failure on ctx (or of the last failed pa_init when ctx is NULL).
 * Valid until the next call on the same context. */
const char* pa_last_error(const pa_ctx* ctx);

/* Synchronise `stream`, then read and clear the context's device status word.
 * Returns PA_OK, PA_ETIMEOUT if a kernel's bounded wait gave up, or PA_ECUDA. */
int pa_sync_status(pa_ctx* ctx, void* stream);

/* pa_sync_status with a host-side deadline: poll `stream` (cudaStreamQuery) for up to
 * timeout_s seconds (0 <= timeout_s <= 86400).  If its work has not finished by then,
 * return PA_ETIMEOUT without touching the status word -- nothing is cancelled, and the
 * caller may wait again or tear down; otherwise as pa_sync_status.  The library's
 * counterpart, on the host, of the bounded device-side waits (the pages describe none).
 * Errors: PA_EINVAL, PA_ETIMEOUT, PA_ECUDA. */
int pa_wait_status(pa_ctx* ctx, void* stream, double timeout_s);

/* Library version string. */
const char* pa_version(void);

/* ---------------------------------------------------------------- partition attention */
typedef struct {
  pa_dtype dtype;            /* PA_BF16 (tensor cores, fp32 accumulate) or PA_F32 (fp32 FMA) */
  int B, H, N, D;            /* D in {64, 128} */
  float scale;               /* softmax scale, normally 1/sqrt(D) */
  const void* q;             /* [B][H][N][D] */
  const void* k;             /* [B][H][N][D] */
  const void* v;             /* [B][H][N][D] */
  int P;                     /* 1..PA_MAX_P */
  const int32_t* part_off;   /* host, P+1 entries */
  int G;                     /* partitions per group, 1..P */
  const uint8_t* fresh;      /* host, QG*KG entries; NULL = every pair fresh */
  void* o_part;              /* [P][B][H][N][D] out: rows of selected pairs written */
  float* lse_part;           /* [P][B][H][N]    out: rows of selected pairs written */
} pa_attn_desc;

/* For every query row i of query group qg and every partition p of a KV group kg with
 * fresh[qg][kg] != 0, write O_p(i) (rounded to dtype, round-to-nearest-even) and
 * LSE_p(i).  Entries of pairs not selected are left untouched.  bf16 runs on tcgen05
 * tensor cores (bf16 operands, fp32 accumulation, P rounded to bf16 for the PV
 * product); f32 runs on fp32 FMA units.  Errors: PA_EINVAL, PA_EALIGN,
 * PA_EUNSUPPORTED, PA_ECUDA. */
int pa_partition_attn(pa_ctx* ctx, const pa_attn_desc* desc, void* stream);

/* ---------------------------------------------------------------- merge with reuse */
typedef struct {
  pa_dtype dtype;
  int B, H, N, D, P, G;
  const int32_t* part_off;   /* host, P+1 entries */
  const void* o_fresh;       /* [P][B][H][N][D] */
  const float* lse_fresh;    /* [P][B][H][N] */
  const void* o_cached;      /* [P][B][H][N][D]; may be NULL only when every pair is fresh */
  const float* lse_cached;   /* [P][B][H][N];    same rule */
  const uint8_t* fresh;      /* host, QG*KG entries; NULL = every pair fresh */
  void* o;                   /* [B][H][N][D] out */
  float* lse;                /* [B][H][N]    out */
  float* w;                  /* [QG][P] out (fused importance of the merged states), or NULL */
  int cached_per_group;      /* 0: o_cached / lse_cached hold per-partition states [P][..];
                                1: they hold one composed state per KV group [KG][B][H][N](D)
                                (see pa_compose_states); w must then be NULL */
} pa_merge_desc;

/* Per row i of query group qg: take the state of partition p from the fresh arrays when
 * fresh[qg][p/G] != 0, else from the cached arrays; write LSE(i), O(i) (fp32 math, O
 * rounded to dtype) and, if w != NULL, overwrite w with the importance of the merged
 * states.  With cached_per_group, a reused KV group contributes its one composed cached
 * state instead of G per-partition states (fewer bytes read per row).  With w != NULL it
 * uses a context workspace of 4*P bytes per 128-row block of each query group of each
 * (b, h) -- about 4*P*B*H*N/128 bytes -- allocated on first need and grown, never shrunk.
 * Errors: PA_EINVAL, PA_EALIGN, PA_EUNSUPPORTED, PA_ENOMEM, PA_ECUDA. */
int pa_merge_states(pa_ctx* ctx, const pa_merge_desc* desc, void* stream);

/* ---------------------------------------------------------------- group compose */
/* Dynamic group compose of cached states (DiTango web summary, Methodology 2, "Dynamic
 * Group Compose": cached states merge recursively into coarser groups with no
 * recomputation).  For every row and every group c of `factor` consecutive partitions,
 * writes the composition of their states: lse_group[c] = ln sum_p exp(lse_part[p]),
 * o_group[c] = sum_p exp(lse_part[p] - lse_group[c]) o_part[p].
 *   o_part [P][B][H][N][D], lse_part [P][B][H][N] in; o_group [C][B][H][N][D],
 *   lse_group [C][B][H][N] out, C = ceil(P / factor).  Partitions of empty state
 *   (-inf) contribute nothing.  Composing G partitions per group gives the cache that
 *   pa_merge_states reads with cached_per_group = 1.
 * Errors: PA_EINVAL, PA_EALIGN, PA_EUNSUPPORTED, PA_ECUDA. */
int pa_compose_states(pa_ctx* ctx, pa_dtype dtype, int B, int H, int N, int D, int P, int factor,
                      const void* o_part, const float* lse_part, void* o_group, float* lse_group,
                      void* stream);

/* ---------------------------------------------------------------- merge without allocation */
/* The same merge (and optional fused importance) as pa_merge_states, for callers that
 * cannot allocate device memory: a process whose memory is owned by another allocator
 * (a framework's caching pool holding the free HBM), or a latency-critical loop that must
 * not stall, since cudaMalloc / cudaFree of a growing workspace synchronise the device.
 * It takes no context (creating one allocates) and allocates nothing: its scratch is a
 * fixed 4 MiB file-scope device array inside libpa, present on every GPU that loads the
 * library until the process exits.  The pages describe no such variant; it has no
 * counterpart there.
 *
 * Arguments, layouts and results are those of pa_merge_states.  The importance scratch
 * needs P * B * H * sum over query groups of ceil(rows / 128) floats; larger requests
 * return PA_EINVAL (use pa_merge_states).  The first call on a device looks up the
 * scratch's device address (cudaGetSymbolAddress) with that device current; make that
 * first call before any stream capture.  Every call shares the one scratch array, whose
 * contents persist between calls (each call writes every scratch entry it reads, so none
 * needs clearing): calls that overlap on the GPU -- on different streams, or from several
 * threads -- race on it.  Errors go to pa_last_error(NULL). */
int pa_merge_states_noalloc(const pa_merge_desc* desc, void* stream);

/* ---------------------------------------------------------------- importance */
/* w[qg][p] = mean over b, h and rows i of qg of exp(lse_part[p][b][h][i] - lse[b][h][i])
 * (0 where lse is -inf).  w is overwritten.  Same workspace rule as pa_merge_states.
 * Errors: PA_EINVAL, PA_EALIGN, PA_ENOMEM, PA_ECUDA. */
int pa_importance(pa_ctx* ctx, int B, int H, int N, int P, int G, const int32_t* part_off,
                  const float* lse_part, const float* lse, float* w, void* stream);

/* ---------------------------------------------------------------- state drift */
/* For every pair (query group qg, partition p) with sel[qg*KG + p/G] != 0:
 *   d2[qg*P + p] = sum over b, h, rows i of qg and channels c of
 *                  (o_new[p][b][h][i][c] - o_ref[p][b][h][i][c])^2,
 *   r2[qg*P + p] = the same sum of o_ref[p][b][h][i][c]^2;
 * 0 for the other pairs.  DiTango, Methodology 1, "Online Prediction": between anchor
 * steps the change of the local states (own KV group, always recomputed) measured against
 * the anchor's cached states estimates how fast the reused states drift; a caller turns
 * d2 / r2 into a relative drift and combines it with the stored importance w.
 *   o_new, o_ref  [P][B][H][N][D] device, dtype (the layout of pa_partition_attn's o_part);
 *                 only the rows of selected pairs are read, so unselected pairs may hold
 *                 anything.  D = 64 or 128.
 *   sel           host uint8[QG*KG]; NULL selects every pair.
 *   d2, r2        device float[QG*P], overwritten.  Sums are taken per 128-row block in
 *                 fp32 and added over blocks in fp64 in a fixed order (deterministic).
 * Uses the context's workspace (2 * P floats per 128-row block of each (b, h); same rule
 * as pa_merge_states).  Errors: PA_EINVAL, PA_EALIGN, PA_EUNSUPPORTED, PA_ENOMEM, PA_ECUDA. */
int pa_state_drift(pa_ctx* ctx, pa_dtype dtype, int B, int H, int N, int D, int P, int G,
                   const int32_t* part_off, const uint8_t* sel, const void* o_new,
                   const void* o_ref, float* d2, float* r2, void* stream);

/* ---------------------------------------------------------------- bounded-wait self-test */
/* Library diagnostics; the pages have no counterpart.  Every pipeline barrier wait in the
 * kernels gives up after a time limit instead of spinning for ever, records PA_ETIMEOUT in
 * the context status word and stops the block.  This call launches a one-block kernel
 * whose two waits (the whole-warp form and the per-thread form) wait on a barrier nothing
 * completes, with a limit of `seconds` (0 < seconds <= 2): both give up within the limit,
 * and a following pa_sync_status returns PA_ETIMEOUT (and clears it), after which the
 * context is usable again.  No fault and no hang are involved.
 * Errors: PA_EINVAL, PA_ECUDA. */
int pa_selftest_wait(pa_ctx* ctx, double seconds, void* stream);

/* ---------------------------------------------------------------- relayout */
/* dst[h][n][:] = src[n][h][:] for the tokens of sequence chunk `chunk` of `n_chunks`
 * (chunk c covers n in [c*ceil(N/n_chunks), min((c+1)*ceil(N/n_chunks), N)));
 * chunk = -1 moves every chunk.  A bit-exact copy: D*elem_bytes must be a multiple of
 * 16 and at most 16384.  Errors: PA_EINVAL, PA_EALIGN, PA_EUNSUPPORTED, PA_ECUDA. */
int pa_relayout_seq2head(pa_ctx* ctx, const void* src, void* dst, int N, int H, int D,
                         int elem_bytes, int n_chunks, int chunk, void* stream);

/* dst[h][dst_tok0 + n][:] = src[n][h][:] for n in [0, n_tok): one sequence piece,
 * sequence-major src [n_tok][H][D], placed at its token offset in a head-major dst
 * [H][dst_tokens][D] (dst_tok0 + n_tok <= dst_tokens).  The receive side of a chunked
 * sequence-parallel all-to-all: each piece arriving from another rank lands in the
 * head-major tensor attention reads -- SwiftFusion, Methodology 2 ("Torus Attention").
 * Bit-exact; same row rules as pa_relayout_seq2head.
 * Errors: PA_EINVAL, PA_EALIGN, PA_EUNSUPPORTED, PA_ECUDA. */
int pa_relayout_seq2head_at(pa_ctx* ctx, const void* src, void* dst, int n_tok, int H, int D,
                            int elem_bytes, int dst_tokens, int dst_tok0, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
