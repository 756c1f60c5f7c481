/*
 * pbs.h - C ABI of libpbs, the sm_100a (B200) implementation of the prefill
 * path of Permuted Block-Sparse Attention (PBS-Attn).
 *
 * Method: "Sparser Block-Sparse Attention via Token Permutation"
 * (arXiv 2510.21270). The five calls below are its five steps:
 *
 *   pbs_score          key importance from the last query block
 *   pbs_permute        segment-local key order, K/V (and Q) gathered by it
 *   pbs_select_blocks  key blocks kept per query block, from pooled scores
 *   pbs_attn_fwd       causal block-sparse attention on the permuted keys
 *   pbs_unpermute      inverse permutation of the output rows
 *   pbs_attn_fwd_unpermute  the last two fused: rows written in place
 *   pbs_attn_fwd_gather     the forward reading K, V through kpos (no K', V')
 *   pbs_attn_fwd_bcast      the forward writing its rows into several
 *                      buffers (the all-gather of a head-sharded output)
 *   pbs_attention_host the whole path on host buffers, copies overlapped
 *   pbs_block_mass, pbs_coverage  diagnostics: attention coverage and
 *                      block-level density
 *
 * Conventions shared by every call
 * --------------------------------
 * - Tensors are dense, row-major, head dim innermost, in DEVICE memory:
 *     Q, O        [batch, hq,  n, d]  bf16
 *     K, V, K', V'[batch, hkv, n, d]  bf16
 *   Base pointers must be 16-byte aligned.
 * - Query head g reads KV head g / (hq / hkv) (grouped-query attention).
 * - Supported: d in {64, 128}, block (B) in {64, 128}, segment (S) a
 *   multiple of B, n a multiple of B (the last segment may be shorter than
 *   S when n is not a multiple of S), hq a multiple of hkv. n == 0 or
 *   batch == 0 is a valid empty call that launches nothing.
 * - scale <= 0 selects the softmax scale sigma = 1/sqrt(d).
 * - The caller owns every buffer, the workspace included; the library never
 *   allocates, frees or keeps a pointer after a call returns.
 * - Calls are asynchronous on the given stream (a cudaStream_t; NULL is the
 *   legacy default stream). Argument errors are returned synchronously and
 *   launch nothing. Errors found by a kernel (a wait that ran out, an index
 *   out of range) are recorded in a per-device error word that
 *   pbs_get_device_status reads. Nothing throws across this ABI.
 * - The calls of the device path (pbs_score, pbs_permute,
 *   pbs_select_blocks, pbs_attn_fwd and its _unpermute and _gather forms,
 *   pbs_unpermute) only enqueue work on the given stream: they neither
 *   synchronise nor allocate, so a sequence of them can be captured into a
 *   CUDA graph (stream capture) and replayed on whatever the captured
 *   buffers hold at replay time; shapes, pointers and the softmax scale are
 *   fixed at capture. The whole path captured that way replays bit for bit
 *   like the calls themselves.
 */
#ifndef PBS_H
#define PBS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *pbs_stream_t; /* same type as cudaStream_t */

typedef struct {
  int batch;   /* b */
  int hq;      /* query heads */
  int hkv;     /* key/value heads, divides hq */
  int n;       /* sequence length N */
  int d;       /* head dimension: 64 or 128 */
  int block;   /* block size B of the block-sparse attention: 64 or 128 */
  int segment; /* permutation segment size S: a multiple of B */
} pbs_shape;

typedef enum {
  PBS_OK = 0,
  PBS_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or mode */
  PBS_ERR_UNSUPPORTED = 2,   /* d or B outside the compiled kernels */
  PBS_ERR_CUDA = 3,          /* a CUDA runtime call failed */
  PBS_ERR_TIMEOUT = 4,       /* a kernel's bounded wait ran out */
  PBS_ERR_DEVICE_ASSERT = 5, /* a kernel found an index out of range */
  PBS_ERR_WORKSPACE = 6      /* workspace smaller than pbs_workspace_bytes */
} pbs_status;

typedef enum {
  PBS_SEL_THRESHOLD = 0,   /* keep blocks until the kept softmax mass >= tau */
  PBS_SEL_TOPK_FRAC = 1,   /* keep max(1, floor(f * (I + 1))) blocks */
  PBS_SEL_ALL = 2,         /* every admissible block */
  PBS_SEL_DENSE_CAUSAL = 3 /* blocks J <= I: plain causal attention */
} pbs_sel_mode;

typedef enum {
  PBS_OP_SCORE = 0,
  PBS_OP_PERMUTE = 1,
  PBS_OP_SELECT = 2,
  PBS_OP_ATTN = 3,
  PBS_OP_UNPERMUTE = 4,
  PBS_OP_HOST_PATH = 5 /* pbs_attention_host */
} pbs_op;

/* Bytes of device workspace the call `op` needs for shape `s` (0 if none). */
size_t pbs_workspace_bytes(pbs_shape s, int op);

/*
 * pbs_score - global key importance from the last query block.
 * Source: gist.science summary of the paper, "Methodik" 3 ("Proxy-
 * Bewertung"): importance is estimated from the last block of queries by
 * mean pooling their attention scores.
 *
 * For each (batch, KV head h) the probe rows are the last B query rows of
 * each of the G = hq/hkv query heads of h's group (G*B rows, positions
 * n-B .. n-1). Each probe row r attends causally over all n keys with
 * logits sigma * q_r . k_j; imp[b, h, j] is the mean over the G*B rows of
 * the softmax probability of key j. Each imp row sums to 1.
 *
 *   q   [batch, hq, n, d] bf16 (only the last B rows of each head are read)
 *   k   [batch, hkv, n, d] bf16
 *   imp [batch, hkv, n] fp32, written
 *   ws  device workspace of at least pbs_workspace_bytes(s, PBS_OP_SCORE)
 */
pbs_status pbs_score(const void *q, const void *k, float *imp, pbs_shape s,
                     float scale, void *ws, size_t ws_bytes, pbs_stream_t st);

/*
 * pbs_score_static - pbs_score for callers that cannot allocate device memory.
 * The paper has no counterpart: this is a deployment variant of pbs_score.
 *
 * Callers such as a plugin inside an inference engine that owns every
 * device allocation (and forbids cudaMalloc), or a latency-critical loop
 * that cannot take cudaMalloc's implicit synchronisation, cannot provide
 * pbs_score's workspace. This call computes the same importance with its
 * scratch in a fixed array of PBS_SCORE_STATIC_SCRATCH_BYTES inside the
 * library, held on every GPU that loads the library until the process
 * exits. It allocates nothing; the caller still passes q, k and imp.
 *
 * - Shapes whose scoring scratch (pbs_workspace_bytes(s, PBS_OP_SCORE))
 *   exceeds the array return PBS_ERR_WORKSPACE and launch nothing.
 * - Arguments are checked first, as pbs_score checks them: an empty shape
 *   returns PBS_OK and a bad one its error, without touching CUDA.
 * - The first call on a device (with that device current) looks up the
 *   array's device address; make it before any stream capture. A failed
 *   lookup returns PBS_ERR_CUDA and is tried again on the next call.
 * - All calls share the array and it keeps the previous call's contents
 *   (nothing in it needs to start at zero). Calls that overlap on the GPU,
 *   from several streams or threads, race on it: serialise them.
 * Other arguments, errors and results: as pbs_score.
 */
#define PBS_SCORE_STATIC_SCRATCH_BYTES (4u << 20)
pbs_status pbs_score_static(const void *q, const void *k, float *imp, pbs_shape s,
                            float scale, pbs_stream_t st);

/*
 * pbs_permute - segment-local key permutation and gather.
 * Source: gist.science summary, "Methodik" 2 (segmented permutation: only
 * inside contiguous segments of S tokens, segment order kept) and 3
 * ("Sortierung": keys sorted by descending global importance inside each
 * segment); sciencestack.ai Lemma 3.1 (K and V permuted together).
 *
 * kpos[b, h, p] = the original index of the key placed at slot p: inside
 * each segment keys are ordered by imp descending, equal values keeping the
 * lower original index first. k_perm[b,h,p] = k[b,h,kpos[p]], likewise v.
 * kbar_sum (optional) receives the fp64 sum of the B rows of each permuted
 * key block: [batch, hkv, n/B, d]. With q non-NULL (permuted-query mode)
 * q_perm[b, g, p] = q[b, g, kpos[b, g/G, p]] for every query head g.
 *
 *   imp         [batch, hkv, n] fp32 (no NaN)
 *   k, v        [batch, hkv, n, d] bf16
 *   q, q_perm   [batch, hq, n, d] bf16, both NULL or both non-NULL
 *   k_perm, v_perm  [batch, hkv, n, d] bf16, written; both NULL: only kpos
 *               and kbar_sum are produced (for pbs_attn_fwd_gather, which
 *               reads K and V through kpos); one NULL is PBS_ERR_INVALID_ARG
 *   kpos        [batch, hkv, n] int32, written
 *   kbar_sum    [batch, hkv, n/B, d] fp64, written if non-NULL
 */
pbs_status pbs_permute(const float *imp, const void *k, const void *v,
                       const void *q, void *k_perm, void *v_perm, void *q_perm,
                       int32_t *kpos, double *kbar_sum, pbs_shape s,
                       pbs_stream_t st);

/*
 * pbs_select_blocks - key blocks to compute for every query block.
 * Source: gist.science summary, "Methodik" 4 ("Block-Auswahl": block
 * importance by mean pooling over the permuted keys); sciencestack.ai
 * Figure 1 caption (blocks of the on-diagonal segment are always computed);
 * skillmd.com "Implementation Steps" (active blocks as a fraction of the
 * block count, at least one).
 *
 * In fp64: qbar = mean of the B rows of query block I of head g, kbar = mean
 * of permuted key block J of KV head g/G, a_IJ = sigma * qbar . kbar for the
 * admissible J (segment(J) <= segment(I)), pi = softmax of a over them.
 * The blocks of I's own segment are always kept. Then
 *   THRESHOLD (param = tau in (0, 1]): earlier-segment blocks are added in
 *     descending a (ties: lower J) while the kept pi mass is < tau;
 *   TOPK_FRAC (param = f in (0, 1]): k = max(1, floor(f * (I + 1))) and the
 *     best max(0, k - own) earlier-segment blocks are added;
 *   ALL: every admissible block; DENSE_CAUSAL: J = 0 .. I.
 *
 *   q_or_qperm  [batch, hq, n, d] bf16: Q, or Q' in permuted-query mode
 *   k_perm      [batch, hkv, n, d] bf16; read only when kbar_sum is NULL
 *   kbar_sum    [batch, hkv, n/B, d] fp64 from pbs_permute, or NULL
 *   blk_idx     [batch, hq, n/B, n/B] int32, written: row (b, g, I) holds
 *               blk_cnt[b, g, I] ascending block indices, the rest untouched
 *   blk_cnt     [batch, hq, n/B] int32, written
 *   blk_mask    [batch, hq, n/B, n/B] uint8 (1 = kept), written if non-NULL
 *   ws          device workspace of pbs_workspace_bytes(s, PBS_OP_SELECT)
 *               bytes: the pooled sums and the score of every admissible
 *               (query block, key block) pair; ALL and DENSE_CAUSAL do not
 *               use it (NULL accepted)
 */
pbs_status pbs_select_blocks(const void *q_or_qperm, const void *k_perm,
                             const double *kbar_sum, pbs_shape s, int mode,
                             float param, float scale, int32_t *blk_idx,
                             int32_t *blk_cnt, uint8_t *blk_mask, void *ws,
                             size_t ws_bytes, pbs_stream_t st);

/*
 * pbs_attn_fwd - causal block-sparse attention over the permuted keys.
 * Source: sciencestack.ai Figure 1 caption (causality kept across segments,
 * on-diagonal segments computed) and Lemma 3.1 / 3.2; gist.science
 * summary, "Methodik" 4 (permuted FlashAttention kernel).
 *
 * For query row i of head g in query block I, the visible keys are the
 * slots p of the kept blocks of (g, I) whose original position kpos[p] is
 * <= the query's original position (qpos[i], or i when qpos is NULL). The
 * output row is the softmax(sigma * q_i . k'_p)-weighted sum of v'_p, in
 * the order of the given queries (permuted order when qpos is non-NULL).
 *
 *   q_or_qperm      [batch, hq, n, d] bf16
 *   k_perm, v_perm  [batch, hkv, n, d] bf16
 *   kpos            [batch, hkv, n] int32, or NULL for the identity
 *   qpos            [batch, hkv, n] int32 (the order of each KV group's
 *                   queries, as from pbs_permute), or NULL = natural order
 *   blk_idx, blk_cnt  as written by pbs_select_blocks; every list must
 *                   hold the query block's own segment so that every row
 *                   sees at least one key
 *   out             [batch, hq, n, d] bf16, written
 *   lse             [batch, hq, n] fp32 natural-log sum of exp, or NULL
 */
pbs_status pbs_attn_fwd(const void *q_or_qperm, const void *k_perm,
                        const void *v_perm, const int32_t *kpos,
                        const int32_t *qpos, const int32_t *blk_idx,
                        const int32_t *blk_cnt, void *out, float *lse,
                        pbs_shape s, float scale, pbs_stream_t st);

/*
 * pbs_attn_fwd_unpermute - pbs_attn_fwd followed by pbs_unpermute, fused:
 * each output row is written straight to its query's original position.
 * Source: skillmd.com "Implementation Steps" (output[argsort(perm)]) and
 * sciencestack.ai Theorem 3.3, as for the two calls it replaces; the fusion
 * itself is this library's (the pages run the two steps separately).
 *
 * Arguments as for pbs_attn_fwd with the queries in permuted order: row p
 * of head g (query q_perm[b, g, p], original position qpos[b, g/G, p]) is
 * written to out[b, g, qpos[b, g/G, p]], and its LSE to lse[b, g, qpos[...]].
 * With qpos NULL this is pbs_attn_fwd. qpos must hold each segment's
 * positions once (as written by pbs_permute); a position outside [0, n) is
 * reported as PBS_ERR_DEVICE_ASSERT and its row is not written. `out` must
 * not overlap q_perm, k_perm or v_perm (PBS_ERR_INVALID_ARG when it is one
 * of them).
 */
pbs_status pbs_attn_fwd_unpermute(const void *q_perm, const void *k_perm,
                                  const void *v_perm, const int32_t *kpos,
                                  const int32_t *qpos, const int32_t *blk_idx,
                                  const int32_t *blk_cnt, void *out, float *lse,
                                  pbs_shape s, float scale, pbs_stream_t st);

/*
 * pbs_attn_fwd_gather - pbs_attn_fwd on the natural K and V, each permuted
 * key read from its original row: key slot p of KV head (b, h) is row
 * kpos[b, h, p] of k and v. The result is bit-identical to pbs_attn_fwd
 * given k_perm = k[kpos], v_perm = v[kpos], without writing or re-reading
 * those copies. Source: as for pbs_attn_fwd; a segment-local permutation
 * (gist.science summary, "Methodik" 2) only decides which rows form each
 * key block, so the forward may fetch them by index. Fetching on the fly is
 * this library's choice (the pages gather before the forward).
 *
 *   q_or_qperm  [batch, hq, n, d] bf16: Q, or Q' in permuted-query mode
 *   k, v        [batch, hkv, n, d] bf16, natural order
 *   kpos        [batch, hkv, n] int32, required: every segment holds a
 *               permutation of its own positions (as from pbs_permute); a
 *               position outside its block's segment is reported as
 *               PBS_ERR_DEVICE_ASSERT and the key's own row is read instead
 *   qpos, blk_idx, blk_cnt, out, lse  as for pbs_attn_fwd
 *   unpermute   nonzero: rows written at qpos as by pbs_attn_fwd_unpermute
 *               (then `out` must not be q_or_qperm, k or v)
 */
pbs_status pbs_attn_fwd_gather(const void *q_or_qperm, const void *k,
                               const void *v, const int32_t *kpos,
                               const int32_t *qpos, const int32_t *blk_idx,
                               const int32_t *blk_cnt, void *out, float *lse,
                               pbs_shape s, float scale, int unpermute,
                               pbs_stream_t st);

/*
 * pbs_attn_fwd_bcast - pbs_attn_fwd (natural query order) whose epilogue
 * writes every output row into n_out buffers at once: the rows of query
 * head g of this call go to head head_offset + g of each buffer. With the
 * KV groups of a sequence split over GPUs, each GPU passes its own output
 * buffer and its peers' (mapped into this device's address space, e.g. a
 * symmetric allocation), and head_offset = its first query head: the
 * forward then also performs the all-gather of the output, its stores to
 * the peers overlapping the rest of its work. Source: as for pbs_attn_fwd;
 * the head-sharded runs follow the pages' tensor-parallel setting (the
 * gist.science summary's experiments at 256K/512K); writing the gathered
 * output from the forward is this library's.
 *
 *   q, k_perm, v_perm, kpos, blk_idx, blk_cnt  as for pbs_attn_fwd (s.hq
 *                   query heads of this call)
 *   outs            HOST array of n_out (1..8) device pointers, each to a
 *                   [batch, hq_total, n, d] bf16 buffer, 16-byte aligned; the
 *                   call only stores to them (heads head_offset ..
 *                   head_offset + s.hq - 1); none may be q, k_perm or v_perm
 *   hq_total        heads of the buffers, >= head_offset + s.hq
 *   head_offset     first head this call writes, >= 0
 * The caller orders the readers after the call on every device that writes
 * into a buffer (e.g. a collective barrier on the same stream).
 * Runs on the two-tile tcgen05 forwards (B = 128, and B = 64 with query
 * tiles of two 64-row blocks); PBS_ERR_UNSUPPORTED where neither launches.
 */
pbs_status pbs_attn_fwd_bcast(const void *q, const void *k_perm,
                              const void *v_perm, const int32_t *kpos,
                              const int32_t *blk_idx, const int32_t *blk_cnt,
                              void *const *outs, int n_out, int hq_total,
                              int head_offset, pbs_shape s, float scale,
                              pbs_stream_t st);

/*
 * pbs_unpermute - inverse permutation of the output rows.
 * Source: skillmd.com "Implementation Steps" (output[argsort(perm)]);
 * sciencestack.ai Theorem 3.3 (permute, attend, un-permute recovers the
 * original result).
 *
 * out[b, g, qpos[b, g/G, p]] = out_perm[b, g, p]. With qpos NULL (natural
 * query order) this is a copy, or nothing when out == out_perm.
 *
 *   out_perm, out  [batch, hq, n, d] bf16 (must not overlap unless equal)
 *   qpos           [batch, hkv, n] int32 or NULL
 */
pbs_status pbs_unpermute(const void *out_perm, const int32_t *qpos, void *out,
                         pbs_shape s, pbs_stream_t st);

/*
 * pbs_attention_host - the whole path (score, permute, select, forward; the
 * queries in natural order) on HOST buffers, with the host-device copies
 * overlapped with the compute.
 * Source: the five steps as documented above; the pipelining is this
 * library's (the pages do not treat host buffers).
 *
 * The work is split by KV group (batch b, KV head h: query heads
 * h*G .. h*G+G-1), in three device slots of the workspace used in turn, and
 * inside a group by query head. On `h2d`: K, V and the last query block of
 * each head (what the scoring and the permutation need), then the query
 * heads in steps. On `compute`: the group's scoring and permutation, then
 * per step, as soon as its heads have arrived, their selection and
 * forward. On `d2h`: each step's output as soon as it is computed. A step
 * is the fewest query heads (a divisor of G) whose forward still fills the
 * device (three waves of CTAs): one head at 128K, the whole group at 32K.
 * So the copies of one group overlap the compute of the previous one, and
 * only one step's copies are exposed at the start and at the end. Work
 * issued later on `compute` is ordered after the last copy to the host, so
 * synchronising `compute` makes `out` valid. `h2d` and `d2h` may be the same
 * stream (the copies then run one after the other) but must differ from
 * `compute` for any overlap. Results equal those of the per-step calls on
 * the same data up to the order of fp32 sums in the importance (the scoring
 * passes split the keys differently for one group than for all).
 *
 *   q, out       host [batch, hq, n, d] bf16 (page-locked memory for
 *                asynchronous copies; pageable memory works, slower)
 *   k, v         host [batch, hkv, n, d] bf16
 *   mode, param  as for pbs_select_blocks
 *   ws           device workspace of pbs_workspace_bytes(s, PBS_OP_HOST_PATH)
 *                bytes (three slots of one KV group's buffers; the size depends
 *                on the current device's SM count through the step size)
 * Returns PBS_ERR_UNSUPPORTED when the scoring step does not support the
 * group shape (see pbs_score).
 */
pbs_status pbs_attention_host(const void *q, const void *k, const void *v,
                              void *out, pbs_shape s, int mode, float param,
                              float scale, void *ws, size_t ws_bytes,
                              pbs_stream_t compute, pbs_stream_t h2d,
                              pbs_stream_t d2h);

/*
 * pbs_block_mass - diagnostics: the exact attention mass of every (query
 * block, key block) pair. Source: sciencestack.ai Figure 2 caption (the
 * attention coverage of a selection is the total attention score its blocks
 * hold) and Figure 4 (block-level density with and without permutation).
 *
 * Query row i (natural order) attends over all n keys: the key in permuted
 * slot p is visible when kpos[p] <= i (kpos NULL: the identity, i.e. the
 * unpermuted sequence). With the dense softmax probabilities P_ip,
 * mass[b, g, I, J] = (1/B) sum over rows i of block I and slots p of block J
 * of P_ip; every (b, g, I) row sums to 1 and entries J past the admissible
 * blocks of I are 0. Two passes over the admissible keys on the tensor cores.
 *
 *   q       [batch, hq, n, d] bf16 (natural order)
 *   k_perm  [batch, hkv, n, d] bf16; kpos [batch, hkv, n] int32 or NULL
 *   mass    [batch, hq, nb, nb] fp32, written
 * Supported: block = 128, hq / hkv <= 4 (else PBS_ERR_UNSUPPORTED).
 */
pbs_status pbs_block_mass(const void *q, const void *k_perm, const int32_t *kpos,
                          float *mass, pbs_shape s, float scale, pbs_stream_t st);

/*
 * pbs_coverage - diagnostics on a block mass (as from pbs_block_mass), per
 * (b, g, I) row: the mass its list of kept blocks holds, and the fewest
 * blocks that hold at least `target` of the row's mass (the blocks in
 * descending mass, counted until their sum reaches the target; nb when the
 * row's total is below it). Sums in fp64, in a fixed order.
 *
 *   mass             [batch, hq, nb, nb] fp32
 *   blk_idx, blk_cnt as written by pbs_select_blocks; needed for coverage
 *   coverage         [batch, hq, nb] fp32, or NULL
 *   blocks_needed    [batch, hq, nb] int32, or NULL; target in (0, 1]
 */
pbs_status pbs_coverage(const float *mass, const int32_t *blk_idx,
                        const int32_t *blk_cnt, double target, float *coverage,
                        int32_t *blocks_needed, pbs_shape s, pbs_stream_t st);

/*
 * Synchronises `st`, returns in *code the current device's error word
 * (a pbs_status; PBS_OK when no kernel reported a problem) and clears it.
 * `detail` (nullable) receives a diagnostic: for PBS_ERR_TIMEOUT the place
 * of the wait that ran out (tens digit: 1 K' loader, 2 V' loader, 3 MMA
 * issuer, 4 softmax; units digit: which wait), else 0.
 */
pbs_status pbs_get_device_status(pbs_stream_t st, int *code, int *detail);

/* Static, human-readable name of a status. */
const char *pbs_status_string(int status);

/* Library version string. */
const char *pbs_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PBS_H */
