/*
 * rr.h — C ABI of the B200 (sm_100a) RRAttention prefill operator.
 *
 * The operator is the one described on the pages of "RRAttention: Dynamic
 * Block Sparse Attention via Per-Head Round-Robin Shifts for Long-Context
 * Inference" (sciencestack page: Abstract, TL;DR, Figure 2 caption for the
 * three stages): a strided pattern search in which each head samples one
 * position per stride, the position shifting from head to head, that picks per
 * query block an adaptive Top-tau set of key blocks (the last query block kept
 * dense), followed by causal block-sparse attention over the selected blocks.
 *
 * Notation: H query heads, Hkv kv heads (H % Hkv == 0, g = H/Hkv), head dim d,
 * sequence length L, block size B, stride S; Ns = L/S, Nb = L/B, r = B/S.
 *
 * Layouts (row-major, batch 1; a batch is a loop over calls):
 *   q, o : [L, H, d]   bf16          k, v : [L, Hkv, d] bf16
 *   count: [H, Nb]     int32         idx  : [H, Nb, Nb] int32
 * Mask format: count[h*Nb+I] in [1, I+1]; idx[(h*Nb+I)*Nb + t], t < count, lists
 * the selected key blocks of row I in strictly ascending order (so J = I, when
 * selected, is last).  Entries at t >= count are not written and not read.
 *
 * Ownership: the caller allocates every buffer (device memory unless stated);
 * the library never allocates or frees device memory.  All device work is
 * enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and the
 * calls return without synchronising, except rr_check_status.
 *
 * Errors: arguments are validated on the host before anything is enqueued:
 * RR_EINVAL (sizes, tau, null pointers), RR_EUNSUPPORTED (d or B outside
 * {64, 128}), RR_EALIGN (a device pointer not 16-byte aligned, or a workspace
 * not 256-byte aligned), RR_ECUDA (a launch failed).  Device-side failures (a
 * bounded wait that ran out) are recorded in a status word inside the
 * workspace; rr_check_status returns them.
 */
#ifndef RR_H_
#define RR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RR_OK = 0,
  RR_EINVAL = 1,
  RR_EUNSUPPORTED = 2,
  RR_EALIGN = 3,
  RR_ECUDA = 4,
  RR_ETIMEOUT = 5,
  RR_ESCRATCH = 6,  /* rr_search_static only: the shape needs more than its static scratch */
  RR_EMASK = 7      /* rr_sparse_attn: a block list outside the mask format (row not computed) */
} rr_status;

/* Bytes of device workspace that rr_search / rr_sparse_attn / rr_attention
 * need for this shape (status word and block masses [H, Nb, Nb] fp32).  The same
 * workspace may be reused by consecutive calls on one stream. */
rr_status rr_workspace_size(int L, int H, int Hkv, int d, int B, int S, size_t* bytes);

/* Pattern search (RRAttention page, Abstract: head round-robin sampling with
 * scores aggregated per stride and an adaptive Top-tau cut; TL;DR: the last
 * query block is always kept; Figure 2 caption: stages 1 and 2).
 *   Sampling: head h samples, in stride i, position p(h,i) = i*S + (h mod S),
 *             on both sides: its query rows and, on its kv head, its keys.
 *   Scores:   s[h,i,j] = q[p(h,i),h] . k[p(h,j),h/g] / sqrt(d) for j <= i,
 *             softmax per sampled row (a causal attention over the head's
 *             strided subsequence, L/S long).
 *   Mass:     summed over the r x r (row, stride) pairs of block (I, J).
 *   Top-tau:  per row I < Nb-1, blocks in (mass desc, J asc) order, shortest
 *             prefix whose share of the row's mass is >= tau (tau >= 1: all).
 *             Row Nb-1 keeps all blocks.  Shares are summed in fixed point
 *             (each mass rounded to a multiple of 2^-31 of the row total, the
 *             total in fp64), so the selection is deterministic; a block whose
 *             running share lies within ~2^-31 of tau may fall either side of
 *             the cut compared with exact arithmetic.
 * In:  q [L,H,d], k [L,Hkv,d] bf16 (device); tau > 0.
 * Out: count [H,Nb], idx [H,Nb,Nb] int32 (device, caller-owned).
 *      mass: NULL, or a device [H,Nb,Nb] fp32 buffer that receives the
 *      unnormalised block mass (entries J <= I; others unspecified).
 * Requires L % B == 0, B % S == 0, d and B in {64, 128}. */
rr_status rr_search(const void* q, const void* k, int L, int H, int Hkv, int d, int B, int S,
                    float tau, int32_t* count, int32_t* idx, float* mass, void* workspace,
                    size_t workspace_bytes, void* stream);

/* Sampling variants of the pattern search.  The pages fix the head rotation of
 * the sampled offset and the stride-level scoring, but leave open three
 * choices, each selectable here (flags may be combined; 0 = rr_search):
 *   RR_VAR_ROTATE        the offset rotates across strides as well as heads:
 *                        head h samples, in stride i, position
 *                        i*S + ((h + i) mod S), on both sides.
 *   RR_VAR_MEAN_KEYS     the key side of stride j is the mean of the stride's S
 *                        keys (fp32, kept as a bf16 hi/lo pair) instead of the
 *                        key at the head's own sampled position: same
 *                        O(L^2/S^2) cost, per-token structure averaged away.
 *   RR_VAR_GQA_MASK      one mask per GQA group: the Top-tau selection runs
 *                        on the sum of the block masses of the H/Hkv query
 *                        heads of a kv head, and every head of the group
 *                        receives that selection (rows of count/idx repeat).
 * Scores, block mass, Top-tau and the last-row protection are those of
 * rr_search.  Out: count [H,Nb], idx [H,Nb,Nb]; mass (optional) receives the
 * per-head block mass [H,Nb,Nb] before any group sum.  The workspace is sized
 * by rr_workspace_size_variant with the same flags (it holds the pooled keys
 * [L/S, Hkv, d] x 2 bf16 with RR_VAR_MEAN_KEYS, the gathered rows
 * [L/S, H, d] bf16 when rotating, the group masses [Hkv, Nb, Nb] fp32 with
 * RR_VAR_GQA_MASK).  Unknown flag bits: RR_EINVAL. */
#define RR_VAR_ROTATE 1u
#define RR_VAR_MEAN_KEYS 2u
#define RR_VAR_GQA_MASK 4u
rr_status rr_workspace_size_variant(int L, int H, int Hkv, int d, int B, int S, unsigned flags,
                                    size_t* bytes);
rr_status rr_search_variant(const void* q, const void* k, int L, int H, int Hkv, int d, int B, int S,
                            float tau, unsigned flags, int32_t* count, int32_t* idx, float* mass,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Causal block-sparse attention over a block mask (RRAttention page, Abstract:
 * only the selected blocks are computed; Figure 2 caption: stage 3).  Query q of block I, head
 * h, attends with scale 1/sqrt(d) to every key k <= q of the blocks listed for
 * (h, I); kv head = h / (H/Hkv).  fp32 softmax and accumulation, bf16 output.
 * In:  q, k, v bf16 (device), count/idx as produced by rr_search (any mask in
 *      the format above is accepted).
 * Out: o [L,H,d] bf16 (device, caller-owned).
 * Mask check: the kernel checks every row it reads against the format (count
 * in [1, I+1], entries strictly ascending inside [0, I]).  A row that breaks it
 * is not computed (its B output rows of head h are written as zeros) and the
 * workspace status word records RR_EMASK with the first such row seen;
 * rr_check_status returns RR_EMASK.  Other rows are unaffected.  The check
 * reads only the count entry and the first count entries of the row's list,
 * so a count outside [1, I+1] is rejected without reading the list. */
rr_status rr_sparse_attn(const void* q, const void* k, const void* v, int L, int H, int Hkv, int d,
                         int B, const int32_t* count, const int32_t* idx, void* o, void* workspace,
                         size_t workspace_bytes, void* stream);

/* rr_search followed by rr_sparse_attn on the same stream.  count/idx are
 * caller-provided device buffers that receive the mask. */
rr_status rr_attention(const void* q, const void* k, const void* v, int L, int H, int Hkv, int d,
                       int B, int S, float tau, int32_t* count, int32_t* idx, void* o,
                       void* workspace, size_t workspace_bytes, void* stream);

/* rr_attention on host-resident tensors, with the host<->device copies
 * pipelined against the kernels item by item.  An item is one kv head with
 * its query heads, except that the first item holds only the first query head
 * and the last item only the last one (the first kernels start sooner, and
 * the O copy that trails the last kernel is smaller).  The copies of item n+2
 * in and of item n out run on `copy_stream` while the search and attention of
 * item n+1 run on `stream` (an item's search starts once its q and k have
 * landed, its attention once v has too).  Results are those of rr_attention bit for
 * bit (each kv head's g query heads are searched with their global head index).
 * In:  q_host [L,H,d], k_host, v_host [L,Hkv,d] bf16, HOST memory (page-locked
 *      for the copies to be asynchronous; pageable memory works but serialises).
 * Out: o_host [L,H,d] bf16 host memory; count [H,Nb], idx [H,Nb,Nb] int32
 *      DEVICE memory.  All caller-owned.
 * Workspace: rr_workspace_size_host bytes of device memory, 256-byte aligned
 * (two slots of one kv head's q, k, v, o, and one kv head's search scratch).
 * Host memory: a small list of the items is allocated per call.
 * Streams: `stream` and `copy_stream` are cudaStream_t; the copy stream first
 * waits for the work already queued on `stream`, and `stream` finally waits for
 * the last copy, so synchronising `stream` covers the whole call (o_host is
 * complete then).  Eight CUDA events are created and released per call; no
 * device memory is allocated.  Validation as rr_attention. */
rr_status rr_workspace_size_host(int L, int H, int Hkv, int d, int B, int S, size_t* bytes);
rr_status rr_attention_host(const void* q_host, const void* k_host, const void* v_host, int L, int H,
                            int Hkv, int d, int B, int S, float tau, int32_t* count, int32_t* idx,
                            void* o_host, void* workspace, size_t workspace_bytes, void* stream,
                            void* copy_stream);

/* Mask diagnostics (the synthetic counterpart of the pattern visualisations,
 * Figures 4 and 5: full-attention ground truth against the RR selection).
 * recall[h*Nb+I] = sum of mass[h,I,J] over the J listed in (count, idx) for row
 * (h, I), divided by the sum of mass[h,I,J] over J <= I.  `mass` is an
 * unnormalised block mass [H, Nb, Nb] fp32 (entries J <= I read), e.g. the
 * `mass` output of rr_search at S = 1, which is the exact full-attention block
 * mass.  All pointers are device memory; recall is [H, Nb] fp32, caller-owned.
 * List entries outside [0, I] are ignored.  Asynchronous on `stream`. */
rr_status rr_mask_recall(const float* mass, const int32_t* count, const int32_t* idx, int H, int Nb,
                         float* recall, void* stream);

/* Dense view of a block mask (debugging and plotting): dense[(h*Nb + I)*Nb + J]
 * = 1 when J is among the first count[h*Nb+I] entries of row (h, I) of idx,
 * else 0.  count [H,Nb] and idx [H,Nb,Nb] int32 as produced by rr_search;
 * dense [H,Nb,Nb] uint8; all device memory, caller-owned.  Entries outside
 * [0, Nb) are ignored, count is clamped to [0, Nb].  Asynchronous on `stream`. */
rr_status rr_mask_to_dense(const int32_t* count, const int32_t* idx, int H, int Nb, uint8_t* dense,
                           void* stream);

/* Decode stage: one new token per sequence, over its KV cache.  The pages name
 * decoding-stage sparsification only as a future extension (sciencestack page,
 * TL;DR); this call carries the prefill rules over to the query at position
 * t = lens[n] - 1 of each sequence n:
 *   Search:   head h scores the cached keys at its own sampled positions
 *             j*S + (h mod S) <= t (the prefill sampling on the key side):
 *             s_j = q . k_j / sqrt(d), softmax over those j, mass of key block
 *             J = sum over its strides, for J <= t/B.
 *   Top-tau:  as rr_search (mass desc, J asc, shortest prefix with share >= tau,
 *             fixed-point sums); the block t/B, which holds the query and the
 *             newest keys, is always kept.  (Prefill keeps the whole last query
 *             block dense; carried over literally that would make every decode
 *             step dense.)
 *   Attention: the query attends, with scale 1/sqrt(d), to every key <= t of
 *             the kept blocks; fp32 softmax and accumulation, bf16 output.
 * In:  q [N,H,d] bf16 (the new tokens' queries); k_cache, v_cache [N,Lmax,Hkv,d]
 *      bf16 with the new tokens' keys and values already written at position
 *      lens[n]-1; lens [N] int32 (device), each in [1, Lmax].
 * Out: count [N,H] int32, idx [N,H,Lmax/B] int32 (kept blocks ascending, valid
 *      below count), o [N,H,d] bf16.  All device memory, caller-owned.
 * Workspace: rr_decode_workspace_size bytes, 256-byte aligned (status word
 * and arrival counters, zeroed by the call; sampled scores, kept-block
 * bitmaps, attention partials, block masses, the prefix of the sequences'
 * block counts).  One call at a time per workspace.
 * Requires Lmax % B == 0, B % S == 0, d and B in {64, 128}, H/Hkv <= 8,
 * Lmax/B <= 4096.  A length outside [1, Lmax] is found on the device: that
 * sequence gets count 0 and a zero output, and rr_check_status returns
 * RR_EINVAL.  Kernels: search CTAs over runs of each (sequence, head)'s
 * sampled keys, the last of a row's CTAs selecting; then one attention CTA
 * per SM over an equal share of all causal key blocks of all sequences and kv
 * heads, which loads each kept K/V block once for every head of its GQA group
 * that kept it; then one CTA per (sequence, kv head) merging the partials. */
rr_status rr_decode_workspace_size(int N, int Lmax, int H, int Hkv, int d, int B, int S, size_t* bytes);
rr_status rr_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* lens, int N, int Lmax,
                    int H, int Hkv, int d, int B, int S, float tau, int32_t* count, int32_t* idx, void* o,
                    void* workspace, size_t workspace_bytes, void* stream);

/* The decode step with the search's sampling variants: flags 0 is rr_decode;
 * RR_VAR_GQA_MASK keeps one list per GQA group, selected (Top-tau plus the
 * current block) on the sum of the group's per-head block masses (each head's
 * normalised to 1), and every head of the group receives it.  A kept block is
 * loaded once for its whole group either way, so with per-head lists the bytes
 * read follow the union of the group's lists, with this flag the group's own
 * selection.  Other flag bits: RR_EINVAL.  Workspace, arguments and outputs as
 * rr_decode. */
rr_status rr_decode_variant(const void* q, const void* k_cache, const void* v_cache, const int32_t* lens, int N,
                            int Lmax, int H, int Hkv, int d, int B, int S, float tau, unsigned flags, int32_t* count,
                            int32_t* idx, void* o, void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, returns the device-side status recorded since the
 * last rr_* call that started on this workspace (RR_OK, RR_ETIMEOUT, RR_EMASK,
 * or RR_EINVAL for a decode cache length out of range), and RR_ECUDA if the
 * stream reports an error. */
rr_status rr_check_status(void* workspace, void* stream);

/* Sets the bound, in nanoseconds, of every device-side wait of later launches
 * (default 2e9).  Returns the previous bound.  Process-wide. */
uint64_t rr_set_wait_limit_ns(uint64_t ns);

/* The pattern search of rr_search, for callers that cannot allocate device
 * memory or hand the library a workspace (for example an operator interface
 * that passes only its input and output tensors, or a process whose device
 * memory is entirely owned by another allocator).  The paper has no
 * counterpart to this entry point; it only changes where the scratch lives.
 *   Scratch: a file-scope device array of 32 MiB inside this library, which
 *   every GPU that loads the library holds until the process exits.  Shapes
 *   whose rr_workspace_size exceeds 32 MiB are rejected with RR_ESCRATCH before
 *   anything is enqueued (e.g. H=32, Hkv=8, d=128, B=128, S=16 fits up to
 *   L=32768; L=65536 and beyond do not).
 *   Allocation: none (no cudaMalloc, cudaFree or allocating library call).  Each
 *   call looks up the array's device address on the current device
 *   (cudaGetSymbolAddress); the first call in a context also loads the
 *   library's device code there, so make that first call before any stream
 *   capture.  Nothing is cached between calls, so a device reset is harmless.
 *   Sharing: every call, on every stream, uses the same array and the array
 *   keeps the last call's contents; calls that overlap on the GPU race, so
 *   serialise them (one stream, or events).
 *   Status: device-side timeouts land in the array's status word, which the
 *   caller cannot name; use rr_search with a workspace when rr_check_status is
 *   needed.
 * Arguments, outputs and validation otherwise as rr_search (mass not offered). */
rr_status rr_search_static(const void* q, const void* k, int L, int H, int Hkv, int d, int B, int S,
                           float tau, int32_t* count, int32_t* idx, void* stream);

/* Static string for a status code. */
const char* rr_status_string(rr_status s);

#ifdef __cplusplus
}
#endif

#endif /* RR_H_ */
