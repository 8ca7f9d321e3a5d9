/*
 * pw.h -- C ABI of the PageWeaver sparse-attention prefill hot path for NVIDIA B200 (sm_100a).
 *
 * The method ("PageWeaver: KV-Guided Query Unions for Sparse Attention", arXiv 2610.11201,
 * Abstract): in dynamic sparse attention every query token selects its own set of KV pages.
 * Queries are assembled into execution groups ("query unions") whose selected page sets add
 * few new pages to the group's union; a group's union pages are loaded once and fill tensor
 * core tiles, while every query keeps exactly its own selected pages (its "original support")
 * and owns its complete output.  A bounded GPU search produces the query IDs of each group;
 * an ID-aware kernel consumes them without materialising reordered Q tensors or cross-page
 * partial outputs.  The AI Radio episode on the paper (paper summary) adds that the search is
 * greedy inside a bounded window and that the execution size g (g = 8 there) is fixed
 * independently of the window W.
 *
 * A complete call is pw_group followed by pw_attn on the same stream.
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers unless the parameter name ends in _host.
 *   - The caller owns and allocates every buffer (pw_groups_size reports the sizes); the
 *     library allocates no memory and never synchronises the stream.  Its one piece of global
 *     state is the fixed scratch array of pw_group_noalloc (below), which the CUDA runtime
 *     places on every device that loads the library.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default).
 *   - The return value reports errors found on the host (arguments, launch failures).
 *     Errors that depend on the data (a selected page outside the query's causal prefix, a
 *     bounded device wait that ran out) are written to *dev_status, an int32 in device
 *     memory: pw_group resets it to PW_OK, and every kernel afterwards records the first
 *     error only.  Kernels never trap; after an error the outputs are defined but not
 *     meaningful.
 *   - Fixed shapes: head dimension 128, page size 64 tokens, FP8 E4M3 K/V, bf16 Q and O.
 *
 * Layouts (row-major, contiguous)
 *   cu_seqlens   int32 [B+1]                 token offsets of the ragged batch; cu[0] = 0
 *   sel_pages    int32 [T, Hkv, kmax]        logical page ids selected by (token, kv head),
 *                                            -1 = unused slot; duplicates are allowed and count
 *                                            once; valid ids are 0 .. own page of the token
 *   Q            bf16  [T, Hq, 128]          query head hq uses kv head hq / (Hq / Hkv)
 *   K_pages      uint8 [n_phys, Hkv, 64, 128] E4M3 codes; logical page p of sequence b lives
 *   V_pages      uint8 [n_phys, Hkv, 64, 128] at physical slot page_table[b * max_pages + p]
 *   page_table   int32 [B, max_pages]
 *   O            bf16  [T, Hq, 128]
 */
#ifndef PW_H
#define PW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pw_status {
    PW_OK = 0,
    PW_ERR_INVALID_ARG = 1,   /* a null pointer, a negative size, inconsistent sizes        */
    PW_ERR_UNSUPPORTED = 2,   /* a shape outside the supported set (see each call)          */
    PW_ERR_BAD_SELECTION = 3, /* a selected page id outside [-1, own page] (device status)  */
    PW_ERR_CAPACITY = 4,      /* a caller buffer is smaller than pw_groups_size requires    */
    PW_ERR_TIMEOUT = 5,       /* a bounded device wait ran out (device status)              */
    PW_ERR_CUDA = 6           /* a CUDA launch or runtime call failed                       */
} pw_status;

/* Execution groups produced by pw_group and consumed by pw_attn.  All array members are
 * device buffers allocated by the caller with the sizes pw_groups_size reports; the scalar
 * members describe them and are filled by the caller (n_groups, union_cap, words, g must
 * equal what pw_groups_size returned for the same arguments).
 *
 *   qids        int32  [n_groups * g]  global token indices of the members, ascending,
 *                                      -1 after the last member
 *   gsize       int32  [n_groups]      members in the group, 1..g
 *   gmeta       int32  [n_groups * 3]  (sequence b, kv head h, window index w)
 *   union_off   int32  [n_groups + 1]  CSR offsets into union_pages
 *   union_pages int32  [union_cap]     logical page ids of each group's union, ascending
 *   bits        uint32 [T * Hkv * words] page bitset of every (token, kv head) selection;
 *                                      pw_attn reads it for the per-query membership masks
 *   sched       int32  [1]             scratch of pw_attn: for a batch of several sequences,
 *                                      the work counter its CTAs take groups from (pw_attn
 *                                      zeroes it on its stream before the kernel, so two
 *                                      pw_attn calls on one pw_groups must not run at the same
 *                                      time; pw_group does not touch it)
 * Groups are ordered by (b, h, w, seed token).
 */
typedef struct pw_groups {
    int32_t *qids;
    int32_t *gsize;
    int32_t *gmeta;
    int32_t *union_off;
    int32_t *union_pages;
    uint32_t *bits;
    int32_t *sched;
    int64_t n_groups;
    int64_t union_cap;
    int32_t words;
    int32_t g;
} pw_groups;

/* Version of this ABI (major * 10000 + minor * 100 + patch). */
int pw_version(void);

/* Human-readable name of a status code (static storage). */
const char *pw_status_string(int status);

/* Sizes, computed on the host without touching the device.
 *   cu_seqlens_host  host copy of cu_seqlens [B+1]
 *   n_groups         number of groups pw_group will emit (a window of n tokens yields
 *                    ceil(n / g) groups, so the count does not depend on the data)
 *   union_cap        capacity needed for union_pages: sum over groups of min(g * kmax, P_b)
 *   words            32-bit words per bitset row: ceil(max_b P_b / 32)
 *   workspace_bytes  device scratch pw_group needs (256-byte aligned start)
 * Supported: 1 <= g <= 32, g * (Hq / Hkv) <= 128 (checked by pw_attn), W a multiple of g with
 * W <= 256, every sequence at most 131072 tokens (words <= 64), union_cap < 2^31.
 * Returns PW_OK, PW_ERR_INVALID_ARG or PW_ERR_UNSUPPORTED. */
pw_status pw_groups_size(const int32_t *cu_seqlens_host, int B, int Hkv, int kmax, int W, int g,
                         int64_t *n_groups, int64_t *union_cap, int32_t *words,
                         size_t *workspace_bytes);

/* Bounded-window greedy grouping (the "bounded GPU search" of the Abstract).
 * Per sequence b and kv head h, tokens are cut into fixed windows [wW, min((w+1)W, len_b)).
 * In a window, while a token is unassigned: the seed is the lowest unassigned token and the
 * group's union U starts as its page set; then, until the group has g members or the window
 * is exhausted, the unassigned token c minimising |S(c) \ U| (pages it adds to the union,
 * lowest token index on ties) joins and U grows by S(c).  W = g reproduces contiguous
 * grouping; g = 1 gives one query per group.
 * Inputs: sel_pages, cu_seqlens (device) and cu_seqlens_host (host copy of the same values).
 * Outputs: every array of *groups (the struct itself is read on the host).
 * workspace: device scratch of at least workspace_bytes from pw_groups_size.
 * Selected ids outside [-1, own page] set PW_ERR_BAD_SELECTION in *dev_status and are ignored.
 */
pw_status pw_group(const int32_t *sel_pages, const int32_t *cu_seqlens,
                   const int32_t *cu_seqlens_host, int B, int Hkv, int kmax, int W, int g,
                   const pw_groups *groups, void *workspace, size_t workspace_bytes,
                   int32_t *dev_status, void *stream);

/* ID-aware union attention (the Abstract's ID-aware kernel).
 * For each group, the union pages are streamed once, in ascending order, through the page
 * table (K and V pages staged by the bulk-copy engine, FP8 decoded on chip); the group tile
 * stacks the G = Hq / Hkv query heads of every member (gsize * G rows, at most 128); S = QK^T
 * and O = PV run on the tensor cores; each row is masked to the pages its own token selected
 * and to keys at or before its position; the softmax is online and exact in fp32; each row
 * writes its complete output O[t, hq, :] = v_scale * softmax(sm_scale * k_scale * q K^T) V,
 * rounded to bf16.  A row with no allowed key writes zeros.
 * Q, K_pages, V_pages, page_table, cu_seqlens and groups (arrays) are read; O is written.
 * T is the token count (rows of Q and O), n_phys the number of physical pages.
 * Supported: Hq % Hkv == 0, groups->g * (Hq / Hkv) <= 128.
 */
pw_status pw_attn(const void *Q, const void *K_pages, const void *V_pages,
                  const int32_t *page_table, int max_pages, int n_phys,
                  const int32_t *cu_seqlens, int B, int64_t T, int Hq, int Hkv,
                  float k_scale, float v_scale, float sm_scale,
                  const pw_groups *groups, void *O, int32_t *dev_status, void *stream);

/* pw_group without a caller-supplied workspace.  The paper has no counterpart: this is a
 * convenience of this library for callers that cannot allocate device memory, e.g. code running
 * where cudaMalloc is not allowed (it can synchronise the device) or a plug-in whose host
 * application owns the whole memory budget and hands it only input and output buffers.
 *
 * Same arguments, outputs and errors as pw_group, minus workspace / workspace_bytes.  The
 * scratch is a fixed device array of PW_NOALLOC_SCRATCH_BYTES inside the library; every GPU that
 * loads the library holds it until the process exits.  The call itself allocates nothing (no
 * cudaMalloc, no cudaFree, no allocating library routine).
 *   - Shapes whose workspace (pw_groups_size) exceeds PW_NOALLOC_SCRATCH_BYTES are rejected
 *     with PW_ERR_CAPACITY before any device work; use pw_group with your own workspace then.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress), so the address stays valid across a device reset.  The first call
 *     on a device also loads the library's device code there; make that first call before any
 *     stream capture.  The stream must belong to the current device.
 *   - All calls on a device share the one array, which keeps the last call's contents.  Nothing
 *     in it needs clearing between calls, but calls that overlap on the GPU (different streams,
 *     no ordering between them) race on it and must not be issued.
 */
#define PW_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

pw_status pw_group_noalloc(const int32_t *sel_pages, const int32_t *cu_seqlens,
                           const int32_t *cu_seqlens_host, int B, int Hkv, int kmax, int W, int g,
                           const pw_groups *groups, int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PW_H */
