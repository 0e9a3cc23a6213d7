/*
 * kda.h — C ABI of libkda.so, a B200 (sm_100a) implementation of the KDA
 * (Kimi Delta Attention) token-mixing recurrence.
 *
 * The operation (Kimi K3 wiki, "Exercices", Q7; the report's eq. 1 as listed
 * on "Ce qui est public et ce qui ne l'est pas"): for every (sequence, head),
 * with state S in R^{dk x dv},
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T q_t,
 *
 * with a per-channel log-decay g_t in [g_min, 0], g_min = -5 ("Exercices",
 * Q8) and an L2-normalised key ("Exercices", Q9). Prefill evaluates it in
 * chunks; the state is carried from chunk to chunk by the KCP pair
 * (cumulative transition, local state) and its composition ("Exercices",
 * Q21-Q22; report eq. 14).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument is DEVICE memory owned by the caller unless the
 *    comment says otherwise (kda_forward_host takes host buffers). The
 *    library never allocates or frees device memory and never synchronises:
 *    work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and the call returns once it is launched. kda_forward_host also
 *    keeps two side streams and eight events per device, made on its first
 *    call there.
 *  - Activations are token-major and contiguous:
 *        q, k, g : [B, T, H, dk]      v, o : [B, T, H, dv]      beta : [B, T, H]
 *    all of the element type `dtype` (o is written in that type too).
 *  - States are fp32, layout [N, H, dv, dk]: element (i, j) of S for unit
 *    (n, h) sits at ((n*H + h)*dv + j)*dk + i (a column of S is contiguous).
 *    Prefill's S_T feeds kda_decode_step's S directly.
 *  - Supported: dk, dv in {32, 64, 128}; chunk in {16, 32, 64}; every pointer
 *    16-byte aligned.
 *  - Preconditions that are documented, not checked: g in [-5, 0],
 *    beta in [0, 1], ||k_t||_2 = 1 (q and k normalised upstream; the kernels
 *    do not renormalise and apply no 1/sqrt(dk) scale). A g below -5 may
 *    overflow the 16-token exponent factorisation.
 *  - Errors: a call whose arguments fail validation returns a non-zero
 *    kda_status and launches nothing. A launch failure returns
 *    KDA_ERR_CUDA. Faults inside a kernel surface at the caller's next
 *    synchronisation of `stream`.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1, /* null required pointer, non-positive or inconsistent sizes */
    KDA_ERR_UNSUPPORTED = 2, /* dk/dv/chunk/dtype/path combination not built            */
    KDA_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned                         */
    KDA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required               */
    KDA_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed               */
    KDA_ERR_TIMEOUT = 6,     /* (device status word) a bounded wait gave up              */
    KDA_ERR_SCRATCH_LIMIT = 7 /* kda_forward_noalloc: more packed sequences than its fixed scratch holds */
} kda_status;

typedef enum { KDA_DTYPE_F32 = 0, KDA_DTYPE_BF16 = 1 } kda_dtype;

/* Pre-operations fused into the kernels (kda_forward_fused, kda_decode_step_fused):
 * KDA_FUSE_NORM_QK: q and k are raw; each (token, head) row of both is L2-normalised
 *   inside the kernel ("Exercices", Q9: I - beta k k^T is a well-conditioned projection
 *   only for ||k||_2 = 1; q is normalised the same way); an all-zero row stays zero.
 * KDA_FUSE_GATE_LOGITS: g holds gate logits x; the log-decay is g_min sigmoid(x) with
 *   g_min = -5, which maps onto [g_min, 0] ("Exercices", Q8). The pages bound g but do
 *   not print its formula; this is the plainest map onto that range. */
typedef enum { KDA_FUSE_NORM_QK = 1, KDA_FUSE_GATE_LOGITS = 2 } kda_fuse;

/* Which prefill kernels kda_forward_ex runs. The tensor cores cover bf16,
 * dk = dv = 128, chunk = 64; the SIMT kernel covers every supported shape.
 * On the tensor cores there are three forms of the same computation. The part
 * of a chunk that does not depend on the state it receives (decayed Grams,
 * triangular solve, W, Ut; "Exercices", Q21: a chunk's KCP pair depends on
 * its own inputs only) is either computed on each unit's serial path or by
 * chunk-parallel producers that hand a 73 KiB record per chunk to the state
 * chains:
 *  - single (TC_SINGLE): one kernel per (sequence, head) computes everything
 *    chunk after chunk; no workspace beyond the packed-batch schedule.
 *  - split (TC_SPLIT): a chunk-parallel kernel writes every chunk's record to
 *    the workspace, then a second kernel carries each unit's state across its
 *    chunks (73 KiB of workspace per chunk per head). For one sequence of 32 or
 *    more heads that leave at least 8 SMs free (and 4 or more chunks), the first kernel
 *    writes the first chunks' records only and the second is a cooperative
 *    launch in which the free SMs write the last ones beside the chains (the
 *    same records and arithmetic, bit for bit; the same workspace). Where a
 *    cooperative launch is not possible, the two-kernel order runs.
 *  - pipe (TC_PIPE): one cooperative launch runs the chains and the producers
 *    at once, the records passing through a ring of 4 per unit; for at most
 *    two thirds of twice the SM count of units (197 on 148 SMs), else
 *    KDA_ERR_UNSUPPORTED. Workspace: about 292 KiB per unit.
 * AUTO and TC run the single form for batches of more than eight units per
 * SM in dense batches, three in packed ones (all SMs are busy and records
 * would only add traffic); otherwise the
 * split form when the workspace holds it, then the pipe form when its ring
 * fits, else the single form (TC returns KDA_ERR_UNSUPPORTED off the
 * tensor-core shapes, AUTO falls back to SIMT); a forced form returns
 * KDA_ERR_WORKSPACE if the workspace is too small
 * (kda_forward_workspace_size_ex gives each path's need). */
typedef enum {
    KDA_PATH_AUTO = 0,
    KDA_PATH_SIMT = 1,
    KDA_PATH_TC = 2,
    KDA_PATH_TC_SINGLE = 3,
    KDA_PATH_TC_SPLIT = 4,
    KDA_PATH_TC_PIPE = 5
} kda_path;

/* Human-readable name of a status code (static string, never NULL). */
const char *kda_status_string(int status);

/* ABI version of this header (bumped when a signature changes). */
int kda_abi_version(void);

/* Name of the CUDA error behind the last KDA_ERR_CUDA this thread received
 * from an entry point (a static string, "none" if there was none). */
const char *kda_last_cuda_error(void);

/*
 * Bytes of device workspace kda_forward needs for these sizes (0 if none):
 * the scratch of the chunked prefill of "Exercices", Q7 with the KCP
 * composition of Q21-Q22. num_seqs is the number of packed sequences when
 * cu_seqlens is used, else B (B == 1 with num_seqs > 1 means packed
 * sequences). On the tensor-core shapes it is what AUTO runs (kda_path): for
 * batches of up to eight (sequence, head) units per SM (dense) or three
 * (packed), the split form's
 * per-chunk records (74,752 bytes per chunk per head; for packed batches
 * counted for at most T / 64 + num_seqs chunks per head, plus the sequences'
 * chunk offsets and a longest-first schedule of up to 2048 sequences); for
 * larger batches, the single form's schedule only. A smaller workspace still
 * works on the tensor cores (see kda_path). The workspace is scratch: its contents on entry do not
 * matter and it may be reused after the stream reaches the end of the call.
 * Returns (size_t)-1 if the sizes are invalid.
 */
size_t kda_forward_workspace_size(int B, int T, int H, int dk, int dv, int chunk,
                                  int num_seqs, int dtype);

/* The workspace kda_forward_ex needs with an explicit path (kda_path): the form
 * that path runs with that workspace; kda_forward_workspace_size is this with
 * KDA_PATH_AUTO. (size_t)-1 if the sizes or the path are invalid. */
size_t kda_forward_workspace_size_ex(int B, int T, int H, int dk, int dv, int chunk,
                                     int num_seqs, int dtype, int path);

/*
 * Chunked prefill with KCP inter-chunk state composition: the recurrence of
 * "Exercices", Q7 evaluated chunk by chunk, the state carried across chunks
 * by the pair composition of Q21-Q22.
 *
 *   q, k, g, v, beta : inputs (layouts above).
 *   S0   : [N, H, dv, dk] fp32 initial states, or NULL for zeros.
 *   o    : [B, T, H, dv] output, dtype.
 *   S_T  : [N, H, dv, dk] fp32 final states, or NULL to skip; may alias S0
 *          (each unit reads its S0 fully before writing its S_T).
 *   B, T, H, dk, dv : sizes; T = 0 is allowed (S_T = S0, nothing else).
 *   chunk : tokens per chunk (16, 32 or 64).
 *   cu_seqlens : NULL for B dense sequences of T tokens (N = B), or device
 *          int32 [num_seqs + 1] offsets of packed sequences (B must be 1,
 *          cu_seqlens[0] = 0, non-decreasing, cu_seqlens[num_seqs] = T;
 *          chunks never straddle sequences; N = num_seqs).
 *   workspace / workspace_bytes : device scratch of at least
 *          kda_forward_workspace_size(...) bytes (may be NULL when that is 0).
 *   dev_status : NULL, or a device int the kernels set to KDA_ERR_TIMEOUT if
 *          a bounded wait gives up (the caller zeroes it and reads it after
 *          synchronising).
 *   stream : cudaStream_t to enqueue on.
 */
int kda_forward(const void *q, const void *k, const void *v, const void *g, const void *beta,
                const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv,
                int chunk, int dtype, const int32_t *cu_seqlens, int num_seqs,
                void *workspace, size_t workspace_bytes, int *dev_status, void *stream);

/* kda_forward with an explicit kernel choice (kda_path). KDA_PATH_TC on a
 * combination the tensor-core kernel does not cover returns
 * KDA_ERR_UNSUPPORTED. */
int kda_forward_ex(const void *q, const void *k, const void *v, const void *g, const void *beta,
                   const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv,
                   int chunk, int dtype, const int32_t *cu_seqlens, int num_seqs,
                   void *workspace, size_t workspace_bytes, int *dev_status, void *stream,
                   int path);

/* kda_forward_ex with fused pre-operations (flags: kda_fuse bits; 0 = kda_forward_ex).
 * Unknown bits return KDA_ERR_INVALID_ARG. The form is chosen as by
 * kda_forward_ex (the split form's record producer and the single form both have
 * a fused variant); KDA_PATH_TC_PIPE with flags returns KDA_ERR_UNSUPPORTED, and
 * where AUTO would run the pipe form the single form runs. */
int kda_forward_fused(const void *q, const void *k, const void *v, const void *g, const void *beta,
                      const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv, int chunk,
                      int dtype, const int32_t *cu_seqlens, int num_seqs, void *workspace,
                      size_t workspace_bytes, int *dev_status, void *stream, int path, int flags);

/* Number of kernel launches one kda_forward_ex call with these arguments
 * enqueues (0 when T = 0 and no state is copied), or -1 if invalid. For AUTO
 * and TC it assumes the workspace kda_forward_workspace_size reports. */
int kda_forward_launches(int B, int T, int H, int dk, int dv, int chunk, int dtype,
                         int has_cu_seqlens, int num_seqs, int path);

/*
 * Prefill of dense batches whose inputs and outputs are in HOST memory.
 * The state is a fixed-size summary of the whole past ("Exercices", Q6), and
 * a part of a sequence acts only on the state it receives ("Exercices", Q21).
 * So the call cuts every sequence into pieces of piece_len tokens and runs
 * each piece as one kda_forward_ex launch from the fp32 state the previous
 * piece left on the device. Piece p's inputs are uploaded while piece p-1
 * runs and piece p-2's outputs are downloaded, on two side streams of the
 * library. With piece_len a multiple of chunk, o and S_T equal those of one
 * kda_forward_ex call over all T tokens bit for bit.
 *
 *   q, k, g : host [B, T, H, dk]; v : host [B, T, H, dv]; beta : host [B, T, H];
 *          all of dtype. Page-locked (pinned) memory lets the copies run
 *          asynchronously and overlap; pageable memory works but serialises.
 *   S0   : host [B, H, dv, dk] fp32, or NULL for zeros.
 *   o    : host [B, T, H, dv] output, dtype. S_T : host [B, H, dv, dk] fp32, or NULL.
 *   piece_len : tokens per piece, a positive multiple of chunk, or 0 for
 *          about T / 8 rounded up to whole chunks.
 *   workspace / workspace_bytes : DEVICE memory, 256-byte aligned, of at least
 *          kda_forward_host_workspace_size(...) bytes: two slots for one
 *          piece's inputs and outputs, the state, and the device prefill's
 *          workspace for one piece (kda_forward_workspace_size of a piece).
 *   dev_status, path : as for kda_forward_ex. stream : the caller's stream;
 *          the launches run on it, and it is made to wait for the last
 *          download, so the host outputs are complete once the stream is.
 * Host buffers and the workspace must stay valid until then. Ownership stays
 * with the caller. Returns KDA_OK, a validation status (nothing enqueued), or
 * KDA_ERR_CUDA (a CUDA call failed; work may have been enqueued). Calls on
 * one device serialise while they enqueue (a mutex); the side streams and
 * events are created on a device's first call and kept until process exit.
 */
size_t kda_forward_host_workspace_size(int B, int T, int H, int dk, int dv, int chunk, int dtype,
                                       int piece_len);
int kda_forward_host(const void *q, const void *k, const void *v, const void *g, const void *beta,
                     const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv,
                     int chunk, int dtype, int piece_len, void *workspace, size_t workspace_bytes,
                     int *dev_status, void *stream, int path);

/*
 * kda_forward_host for a packed batch (the cu_seqlens layout of kda_forward:
 * q, k, g [T, H, dk], v, o [T, H, dv], beta [T, H], S0 / S_T [num_seqs, H, dv,
 * dk], all in HOST memory; cu_seqlens a HOST int32 array [num_seqs + 1] with
 * cu_seqlens[0] = 0, non-decreasing, cu_seqlens[num_seqs] = T). The flat token
 * axis is cut into pieces of about piece_len tokens (0: about T / 8), each cut
 * moved down onto the chunk grid of the sequence it falls in, so every part of
 * a sequence starts at one of its own chunk boundaries; piece p is one packed
 * kda_forward_ex launch over the sequences it touches, from and to their fp32
 * states in a device buffer (in place). Uploads, launches and downloads
 * overlap as in kda_forward_host. Results equal one device call's up to
 * rounding (a piece may run a different tensor-core form than the whole batch).
 * workspace: at least kda_forward_host_varlen_workspace_size(...) bytes,
 * 256-byte aligned. Other arguments and errors as kda_forward_host.
 */
size_t kda_forward_host_varlen_workspace_size(int T, int H, int dk, int dv, int chunk, int dtype,
                                              const int32_t *cu_seqlens, int num_seqs, int piece_len);
int kda_forward_host_varlen(const void *q, const void *k, const void *v, const void *g, const void *beta,
                            const float *S0, void *o, float *S_T, int T, int H, int dk, int dv, int chunk,
                            int dtype, const int32_t *cu_seqlens, int num_seqs, int piece_len, void *workspace,
                            size_t workspace_bytes, int *dev_status, void *stream, int path);

/*
 * kda_forward without a workspace argument, for callers that cannot allocate
 * device memory: engines that reserve all device memory in their own pools at
 * start-up and treat any other allocation as an error, hosts that hand a
 * library raw device pointers but no allocator, and latency-critical paths
 * where an allocation could block. (The Kimi K3 pages have no counterpart; it
 * is an interface convenience, not part of the method.)
 *
 * Same arguments and results as kda_forward, minus workspace. The only
 * scratch the computation uses, the longest-first schedule of a packed batch,
 * lives in a fixed array of this library's own device memory: 2048 int32
 * (8 KiB), held by every GPU that loads the library until the process exits.
 * Hence the limit: a packed batch (cu_seqlens != NULL) of more than 2048
 * sequences returns KDA_ERR_SCRATCH_LIMIT and launches nothing; dense batches
 * have no limit. This entry point itself allocates nothing.
 *
 * The array belongs to the current device: make the device that owns the
 * tensors current before the call, and pass a stream of that device. Each call
 * made outside a stream capture looks up the array's device address (with that
 * device current), so an address never outlives a context reset; a call made
 * while the stream is being captured reuses the address from the last call on
 * that device outside a capture, so make one call on each device before any
 * stream capture. Every call shares the one array per device and leaves its
 * contents behind (each call overwrites what it reads, so stale contents are
 * harmless); calls that overlap on the GPU race on it, so do not run two at
 * once on one device.
 */
int kda_forward_noalloc(const void *q, const void *k, const void *v, const void *g,
                        const void *beta, const float *S0, void *o, float *S_T, int B, int T,
                        int H, int dk, int dv, int chunk, int dtype, const int32_t *cu_seqlens,
                        int num_seqs, int *dev_status, void *stream);

/*
 * kda_forward on B dense sequences (no cu_seqlens) that also saves the state
 * every snap_every tokens, for a prefix cache on a hybrid model ("Exercices",
 * Q26: a prefix can only be reused where the KDA state was saved, and the
 * state is large, so it is saved at coarse boundaries).
 *
 *   snap_every : tokens between snapshots, a positive multiple of chunk.
 *   S_snap     : fp32 [B, T / snap_every, H, dv, dk]: slot p of sequence b is
 *                the state after its first (p + 1) snap_every tokens, in the
 *                S0 layout of one sequence (it can be passed back as S0 to
 *                resume from that prefix). May be NULL when T < snap_every.
 * Other arguments, results and errors as kda_forward_ex. The workspace decides
 * the tensor-core form as there: with kda_forward_workspace_size_ex(..., path)
 * bytes the split form runs (its chains store the snapshots; dense batches of
 * up to one (sequence, head) unit per SM), with NULL, 0 the single form.
 * KDA_PATH_TC_PIPE is refused (KDA_ERR_UNSUPPORTED), and so is
 * KDA_PATH_TC_SPLIT for more units than SMs.
 */
int kda_forward_snapshots(const void *q, const void *k, const void *v, const void *g, const void *beta,
                          const float *S0, void *o, float *S_T, float *S_snap, int snap_every, int B, int T,
                          int H, int dk, int dv, int chunk, int dtype, void *workspace, size_t workspace_bytes,
                          int *dev_status, void *stream, int path);

/*
 * Segment-parallel prefill for long sequences with few heads (KCP scan, after
 * "Exercices", Q21-Q22 and the 4-rank scan of the pages' check script).
 *
 * Same results as kda_forward on B dense sequences of T tokens (no cu_seqlens),
 * computed differently: each sequence is cut into P = ceil(T / seg_len)
 * segments that run as independent (segment, head) units. Pass A computes each
 * segment's transition M_p (the recurrence from S = I with zero values), pass
 * B its local state S~_p (from S = 0), an fp32 scan composes
 * S_in,p+1 = M_p S_in,p + S~_p from S_in,0 = S0 (its last value is S_T), and
 * pass C replays every segment from S_in,p to write o. The passes read the
 * inputs three times and add a d x d product per segment, so this only pays
 * when (sequences x heads) is well below the SM count and T is long.
 *
 *   seg_len : tokens per segment, a positive multiple of chunk. With P = 1
 *             the call is kda_forward_ex.
 *   workspace / workspace_bytes : device scratch of at least
 *             kda_forward_segmented_workspace_size(...) bytes: for P > 1,
 *             3 x B P H x 64 KiB of fp32 states at d = 128 plus a few bytes per
 *             segment. Scratch only; contents on entry do not matter.
 *   path    : kda_path, as in kda_forward_ex.
 * Other arguments, layouts and errors as kda_forward (S_T may alias S0).
 */
size_t kda_forward_segmented_workspace_size(int B, int T, int H, int dk, int dv, int chunk, int dtype,
                                            int seg_len);
int kda_forward_segmented_launches(int B, int T, int H, int dk, int dv, int chunk, int dtype, int seg_len,
                                   int path);
int kda_forward_segmented(const void *q, const void *k, const void *v, const void *g, const void *beta,
                          const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv, int chunk,
                          int dtype, int seg_len, void *workspace, size_t workspace_bytes, int *dev_status,
                          void *stream, int path);

/*
 * kda_forward_segmented for a packed batch (the cu_seqlens layout of kda_forward:
 * q, k, g [1, T, H, dk], v, o [1, T, H, dv], beta [1, T, H], num_seqs sequences
 * at device offsets cu_seqlens[0..num_seqs], S0 / S_T [num_seqs, H, dv, dk]).
 * Every sequence longer than seg_len is cut into ceil(len / seg_len) segments
 * starting at multiples of seg_len from its first token; shorter ones (empty
 * ones included) are one segment each and go through the same passes as
 * ordinary units. The segment table is built on the device from cu_seqlens
 * (the lengths need not be known on the host): the workspace is sized for the
 * bound T / seg_len + num_seqs on the number of segments. With T <= seg_len
 * no sequence is cut and the call is kda_forward_ex with cu_seqlens.
 *
 *   seg_len : tokens per segment, a positive multiple of chunk.
 *   workspace / workspace_bytes : at least
 *             kda_forward_segmented_varlen_workspace_size(...) bytes.
 *   path    : kda_path, as in kda_forward_ex.
 * Other arguments, results and errors as kda_forward with cu_seqlens.
 */
size_t kda_forward_segmented_varlen_workspace_size(int T, int H, int dk, int dv, int chunk, int dtype, int num_seqs,
                                                   int seg_len);
int kda_forward_segmented_varlen_launches(int T, int H, int dk, int dv, int chunk, int dtype, int num_seqs,
                                          int seg_len, int path);
int kda_forward_segmented_varlen(const void *q, const void *k, const void *v, const void *g, const void *beta,
                                 const float *S0, void *o, float *S_T, int T, int H, int dk, int dv, int chunk,
                                 int dtype, const int32_t *cu_seqlens, int num_seqs, int seg_len, void *workspace,
                                 size_t workspace_bytes, int *dev_status, void *stream, int path);

/*
 * One decode step: one new token for each of N requests, states in place.
 * Same recurrence with T = 1 ("Exercices", Q4: decode is bound by memory
 * bandwidth; each state is read and written exactly once).
 *
 *   q, k, g : [N, H, dk];  v : [N, H, dv];  beta : [N, H]   (dtype)
 *   S       : [N, H, dv, dk] fp32, read and overwritten in place.
 *   o       : [N, H, dv] output, dtype.
 */
int kda_decode_step(const void *q, const void *k, const void *v, const void *g,
                    const void *beta, float *S, void *o, int N, int H, int dk, int dv,
                    int dtype, void *stream);

/*
 * The pieces of the segment-parallel prefill, for callers that place the
 * segments themselves (one segment per GPU: context parallelism, after the
 * pages' 4-rank scan).
 *
 * kda_segment_pair: the KCP pair of each of B dense sequences of T tokens
 * ("Exercices", Q21-Q22): M [B, H, dk, dk], the transition (the recurrence
 * run from S = I with zero values; stored like a state with dv = dk: element
 * (i, a) of M at a * dk + i), and Z [B, H, dv, dk], the local state (from
 * S = 0). fp32. Sizes, dtypes and path as kda_forward_ex.
 *
 * kda_kcp_scan: for B sequences of P consecutive segments with pairs
 * M [B, P, H, dk, dk] and Z [B, P, H, dv, dk] (each segment's pair in the
 * layout above) and incoming states S0 [B, H, dv, dk] (NULL: zeros), writes
 * S_in [B, P, H, dv, dk], the incoming state of every segment
 * (S_in,0 = S0, S_in,p+1 = M_p S_in,p + Z_p, fp32), and S_T [B, H, dv, dk]
 * (NULL to skip), the state after the last segment.
 */
int kda_segment_pair(const void *q, const void *k, const void *v, const void *g, const void *beta, float *M,
                     float *Z, int B, int T, int H, int dk, int dv, int chunk, int dtype, int *dev_status,
                     void *stream, int path);
int kda_kcp_scan(const float *S0, const float *M, const float *Z, float *S_in, float *S_T, int B, int P, int H,
                 int dk, int dv, void *stream);

/* kda_decode_step with fused pre-operations (flags: kda_fuse bits; 0 = kda_decode_step). */
int kda_decode_step_fused(const void *q, const void *k, const void *v, const void *g, const void *beta,
                          float *S, void *o, int N, int H, int dk, int dv, int dtype, void *stream, int flags);

/*
 * Multi-token decode with speculative acceptance ("Exercices", Q27: the state
 * after an accepted prefix of draft tokens is determined by those tokens'
 * inputs, so only the inputs are kept, the recurrence is replayed on chip and
 * the verified state is written back).
 *
 * For each request n, T tokens are applied in order to its states, each as
 * one kda_decode_step; o receives all T outputs (when o is not NULL) and the
 * state after the first n_accept[n] tokens is written back in place
 * (n_accept NULL: all T; 0: S[n] is left untouched). Every state is read
 * once and written at most once, whatever T is.
 * Typical use: verify T draft tokens with n_accept all zero (outputs only),
 * then commit with the accepted counts and o = NULL.
 * A request with outputs and nothing accepted, T <= 16, is computed in the
 * chunked form ("Exercices", Q21-Q22, applied to the T tokens): two dot
 * products per token with every state column, then a T x T triangular
 * system per column; the results equal the sequential steps' up to rounding.
 *
 *   q, k, g : [N, T, H, dk];  v, o : [N, T, H, dv];  beta : [N, T, H]   (dtype)
 *   S        : [N, H, dv, dk] fp32, read, and written where n_accept > 0.
 *   n_accept : device int32 [N] (values clamped to [0, T]) or NULL.
 *   T        : 1..64 (KDA_ERR_UNSUPPORTED above).
 *   dev_status : NULL, or a device int set to KDA_ERR_TIMEOUT if a bounded
 *          wait for the state's staging copies gives up (the outputs and the
 *          states of that request and head are then left unwritten).
 */
int kda_decode_multi(const void *q, const void *k, const void *v, const void *g, const void *beta, float *S,
                     void *o, const int32_t *n_accept, int N, int T, int H, int dk, int dv, int dtype,
                     int *dev_status, void *stream);

/*
 * Diagnostic: one CTA waits, through the same bounded-wait helpers the
 * tensor-core prefill uses, on an mbarrier that nothing arrives on (every wait
 * on a copy or an MMA) and then on a flag in global memory that nothing sets
 * (a chain waiting for a record produced beside it). After max_cycles SM clocks
 * (1 .. 4e9) each wait gives up. dev_status is 4 device ints, 16-byte aligned:
 * [0] receives KDA_ERR_TIMEOUT from the mbarrier wait, [1] is the flag (the
 * caller sets it to zero), [2] receives KDA_ERR_TIMEOUT from the flag wait.
 * Nothing faults or hangs and the stream stays usable; used to test failure
 * reporting without a GPU fault.
 */
int kda_selftest_wait_timeout(int *dev_status, long long max_cycles, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
