/*
 * hhr.h -- C ABI of the B200 (sm_100a) library for the decode-time retrieval
 * path of "HHR: Hierarchical Hash Retrieval for Efficient LLM Generation"
 * (arXiv 2610.01230).
 *
 * What the calls compute (sections of that paper):
 *   GKR, §3.3.1: rotated keys and queries k~ = k R, q~ = q R (Eq. 4); per page
 *     of keys, the per-dimension minimum l and maximum u of the rotated keys
 *     (definition under Eq. 3); the page logit upper bound
 *     U = sum_j max(q~_j l_j, q~_j u_j) (Eq. 3); retention of high-bound pages.
 *   LHP, §3.3.2: projection z = x W (Eq. 10), binary codes c = sign(z) used at
 *     inference (text after Eq. 10; §3.1 Eq. 1), Hamming distance between the
 *     query code and each key code computed with XOR + popcount (§3.1 Eq. 2,
 *     §1), and selection of the closest keys (Top-K ratio, §4.1).
 *   Attention over the selected keys (§1: attention is computed on the keys
 *     the hash retrieval selects).
 *
 * Where the paper leaves a step open, the library takes these readings:
 *   - Page metadata is bf16: the minimum rounded toward -inf, the maximum
 *     toward +inf, so Eq. 3 stays an upper bound of every logit in the page.
 *   - A projection that is exactly 0 gives code bit 0.
 *   - W applies to the unrotated key/query (z = x W, as Eq. 10 writes it).
 *   - GQA: KV head g serves query heads g*r .. g*r+r-1 (r = Hq/Hkv).  A page's
 *     score is the max over those heads of Eq. 3, a token's distance the min
 *     over those heads of Eq. 2.
 *   - The retention threshold c_h of §3.3.1 is a page budget P: the P pages
 *     with the largest score are kept, ties to the lower page index.
 *   - The k tokens of the kept pages with the smallest distance are selected,
 *     ties to the lower token index.  Nothing else is forced in.
 *   - Attention uses the original keys (Eq. 4 leaves logits unchanged) and the
 *     scale the caller passes (usually 1/sqrt(d)).
 *   Two of these readings have a variant, chosen per call by hhr_dims.flags:
 *   - HHR_FLAG_META_F32: page metadata is float32, the extrema exactly as
 *     computed from the float32 rotated keys (no rounding; twice the bytes).
 *   - HHR_FLAG_GQA_SUM: a token's distance is the sum over the group's heads
 *     of Eq. 2 (range 0 .. r*bits) instead of the min.
 *
 * Conventions common to every call
 *   Memory.  The caller owns every buffer.  Pointers documented as "device"
 *     must address CUDA device memory of the current device.  The library
 *     allocates nothing, frees nothing and keeps no pointer after a call
 *     returns.
 *   Streams.  `stream` is a cudaStream_t (NULL: the legacy default stream).
 *     Device work is enqueued on it and the call returns without waiting.
 *     The decode kernels are launched as programmatic dependents of the
 *     preceding kernel on the stream: they may become resident early but
 *     wait for that kernel's completion before touching memory, so stream
 *     order is kept.
 *   Errors.  Every call returns an hhr_status.  Arguments are checked on the
 *     host first; on any return other than HHR_OK or HHR_ERR_CUDA nothing was
 *     enqueued.  HHR_ERR_CUDA reports a failed launch (cudaGetLastError).
 *   Waits.  Decode kernels synchronise the CTAs that share one (sequence, KV
 *     head) through counters in the workspace.  Every such wait gives up after
 *     a bounded number of clock cycles (about one second), records
 *     HHR_ERR_TIMEOUT in the workspace status word and ends the kernel; read it
 *     with hhr_read_status().  The launch is cooperative, so the CTAs of a
 *     launch are co-resident and the wait ends normally.
 *   Layouts (dense, row-major, no padding; bf16 = 16-bit brain float):
 *     K, V      bf16 [B][Hkv][n_cap][d]          keys / values (KV cache)
 *     codes     u32  [B][Hkv][n_cap][bits/32]    bit t of a key's code is bit
 *                                                t%32 of word t/32
 *     meta      bf16 [B][Hkv][ceil(n_cap/page)][2][d]  (f32 with HHR_FLAG_META_F32)
 *                    [p][0][j]: lower bound of dimension j over page p
 *                    [p][1][j]: upper bound of dimension j over page p
 *     R         f32  [Hkv][d][d]                 k~[j] = sum_i k[i] R[i][j]
 *     W         f32  [Hkv][d][bits]              z[t]  = sum_i x[i] W[i][t]
 *     q         bf16 [B][Hq][d]
 *     page_idx  i32  [B][Hkv][P]                 ascending, then -1
 *     tok_idx   i32  [B][Hkv][k]                 ascending, then -1
 *     n_sel     i32  [B][Hkv]                    tokens selected
 *     out       f32  [B][Hq][d]
 *   Page p of a (sequence, KV head) holds tokens [p*page, (p+1)*page).  With
 *   n_valid valid tokens there are ceil(n_valid/page) pages; the last one may
 *   be partial and only its valid tokens count.
 *   Supported sizes: d == 128; bits in {128, 256}; page in {1, 2, 4, ..., 64};
 *   Hq % Hkv == 0 with Hq/Hkv in {1, 2, 4, 8}; B, Hkv >= 1; n_cap >= 1 and
 *   ceil(n_cap/page) <= HHR_MAX_PAGES.  Other sizes return HHR_ERR_UNSUPPORTED.
 */
#ifndef HHR_H_
#define HHR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum hhr_status {
  HHR_OK = 0,
  HHR_ERR_INVALID_ARG = 1, /* null pointer, negative or inconsistent size    */
  HHR_ERR_UNSUPPORTED = 2, /* valid but outside the supported sizes above    */
  HHR_ERR_WORKSPACE = 3,   /* workspace pointer null or smaller than needed  */
  HHR_ERR_CUDA = 4,        /* a CUDA call or kernel launch failed            */
  HHR_ERR_TIMEOUT = 5      /* a bounded inter-CTA wait ran out (device flag) */
} hhr_status;

/* Largest number of pages per (sequence, KV head) a decode call accepts. */
#define HHR_MAX_PAGES 16384

/* hhr_dims.flags: variants of two readings (see the top of this file). */
#define HHR_FLAG_META_F32 1  /* meta is f32, unrounded extrema               */
#define HHR_FLAG_GQA_SUM 2   /* token distance = sum over the group's heads  */
#define HHR_FLAG_SIMT_BOUNDS 4 /* Eq. 3 on the CUDA cores instead of the tensor
                                  cores (bf16 metadata; same results up to
                                  float32 rounding; for comparison)           */

typedef struct hhr_dims {
  int32_t B;     /* sequences                                   */
  int32_t Hq;    /* query heads                                 */
  int32_t Hkv;   /* key/value heads                             */
  int32_t d;     /* head dimension (128)                        */
  int32_t bits;  /* code length b (128 or 256)                  */
  int32_t page;  /* tokens per page S                           */
  int32_t n_cap; /* KV-cache capacity per (sequence, KV head)   */
  int32_t flags; /* 0, or an OR of the HHR_FLAG_* above          */
} hhr_dims;

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t hhr_version(void);

/* Static English text for a status code (never NULL). */
const char* hhr_status_string(int32_t status);

/*
 * Key encoding for keys [n_begin, n_end) of every (sequence, KV head):
 * rotation (Eq. 4), per-page extrema (under Eq. 3) and projection + sign
 * (Eq. 10, Eq. 1).
 *   K     device, read:  bf16 keys, layout above.
 *   R, W  device, read:  f32 rotation / projection, layout above.
 *   codes device, write: codes of keys [n_begin, n_end); other keys untouched.
 *   meta  device, read+write: every page that holds a key of [n_begin, n_end)
 *         is updated.  A page whose first key is below n_begin must already
 *         hold the bounds of its keys [page start, n_begin) (from an earlier
 *         call); the new keys are merged into them (min / max), which gives
 *         the same bytes as encoding the page in one call.  A page starting at
 *         or after n_begin is overwritten.
 * Requires 0 <= n_begin <= n_end <= n_cap; n_begin == n_end enqueues nothing.
 * Keys are encoded to float32 accuracy: the products run on the tensor cores
 * with each f32 weight entered as three bf16 terms whose sum is exactly the
 * weight (so every product with a bf16 key is exact) and f32 accumulation.
 * The kernel's internal pipeline waits are bounded (about one second); one
 * that runs out abandons the call and sets a sticky HHR_ERR_TIMEOUT, read
 * with hhr_encode_status().
 */
int32_t hhr_encode_keys(const hhr_dims* dims, const void* K, const float* R, const float* W,
                        int32_t n_begin, int32_t n_end, uint32_t* codes, void* meta,
                        void* stream);

/*
 * Waits for `stream`, returns the sticky status of the key-encoding kernels
 * on the current device (HHR_OK, or HHR_ERR_TIMEOUT after an abandoned
 * hhr_encode_keys) and clears it.  Returns HHR_ERR_CUDA if the copy or the
 * wait fails.  No counterpart in the paper: it reports the kernel's bounded
 * waits.
 */
int32_t hhr_encode_status(void* stream);

/*
 * Bytes of device workspace hhr_select / hhr_sparse_attend / hhr_decode_step
 * need for these dims and budgets (P pages, k tokens).  The workspace must be
 * zero-filled once before its first use; the library leaves it in that state
 * after every call that completes without HHR_ERR_TIMEOUT.  One workspace
 * must not be used by two calls that may run at the same time.
 * Returns 0 for invalid dims.
 */
size_t hhr_workspace_size(const hhr_dims* dims, int32_t P, int32_t k);

/*
 * Retrieval for one decode step (GKR then LHP) for every (sequence, KV head):
 * query rotation and codes, page bounds of the ceil(n_valid/page) pages
 * (Eq. 3, max over the group), the P best pages, Hamming distances of every
 * valid token of those pages (Eq. 2, min over the group; the sum with
 * HHR_FLAG_GQA_SUM), and the k closest tokens.
 *   q        device, read:  bf16 [B][Hq][d].
 *   R, W     device, read:  as for hhr_encode_keys.
 *   codes, meta device, read: encoded keys [0, n_valid).
 *   n_valid  valid keys per (sequence, KV head), 0 <= n_valid <= n_cap.
 *   P, k     budgets, >= 1.  When fewer pages / candidate tokens exist, all
 *            are kept and the rest of the output row is -1.
 *   page_idx, tok_idx, n_sel device, write (layouts above).
 *   dbg_U    device, write, nullable: f32 [B][Hkv][ceil(n_valid/page)] group
 *            page bounds.
 *   dbg_D    device, write, nullable: i32 [B][Hkv][P*page] group distance of token
 *            page_idx[slot]*page + t at [slot*page + t]; -1 for empty slots and
 *            tokens >= n_valid.
 *   workspace device, read+write: at least hhr_workspace_size(dims, P, k) bytes.
 */
int32_t hhr_select(const hhr_dims* dims, const void* q, const float* R, const float* W,
                   const uint32_t* codes, const void* meta, int32_t n_valid, int32_t P,
                   int32_t k, int32_t* page_idx, int32_t* tok_idx, int32_t* n_sel,
                   float* dbg_U, int32_t* dbg_D, void* workspace, size_t ws_bytes,
                   void* stream);

/*
 * Softmax attention of every query head over the tokens its KV group
 * selected: out[b][h] = sum_i softmax_i(scale * q[b][h].K[b][g][tok_i]) V[b][g][tok_i]
 * over the first n_sel[b][g] entries of tok_idx[b][g] (row stride k), with
 * float32 accumulation of the bf16 inputs.  A group with n_sel == 0 gets zeros.
 *   q, K, V  device, read; tok_idx, n_sel device, read (values < n_cap,
 *            0 <= n_sel <= k); out device, write.
 */
int32_t hhr_sparse_attend(const hhr_dims* dims, const void* q, const void* K, const void* V,
                          const int32_t* tok_idx, const int32_t* n_sel, int32_t k,
                          float scale, float* out, void* workspace, size_t ws_bytes,
                          void* stream);

/*
 * Dense decode attention, the comparator the paper measures HHR against
 * (§4.3 "Context Length", Fig. 7: decode speed of HHR over full attention):
 * out[b][h] = sum_n softmax_n(scale * q[b][h].K[b][g][n]) V[b][g][n] over
 * every key n < n_valid of the head's KV group g, float32 accumulation of the
 * bf16 inputs.  n_valid == 0 gives zeros.  Same kernels and merge as
 * hhr_sparse_attend, over contiguous key ranges (each CTA one range).
 *   q, K, V  device, read; out device, write (layouts above).
 *   n_valid  0 <= n_valid <= n_cap.
 *   workspace as for hhr_sparse_attend (hhr_workspace_size(dims, 1, 1)).
 */
int32_t hhr_dense_attend(const hhr_dims* dims, const void* q, const void* K, const void* V,
                         int32_t n_valid, float scale, float* out, void* workspace,
                         size_t ws_bytes, void* stream);

/*
 * One fused decode step: hhr_select followed by hhr_sparse_attend, in a
 * single launch.  Arguments as for those two calls.
 */
int32_t hhr_decode_step(const hhr_dims* dims, const void* q, const float* R, const float* W,
                        const uint32_t* codes, const void* meta, const void* K, const void* V,
                        int32_t n_valid, int32_t P, int32_t k, float scale, int32_t* page_idx,
                        int32_t* tok_idx, int32_t* n_sel, float* out, void* workspace,
                        size_t ws_bytes, void* stream);

/*
 * hhr_decode_step for a caller whose query and output live in host memory:
 * copies q_host (bf16 [B][Hq][d]) into the device buffer q, runs the step,
 * copies out (f32 [B][Hq][d]) back into out_host and waits for `stream`
 * before returning (the only blocking decode call).  Host buffers should be
 * pinned (page-locked) for the copies to be asynchronous DMA.  Other
 * arguments as for hhr_decode_step; every check is made before anything is
 * enqueued.  The paper has no counterpart: it is the end-to-end form of the
 * decode step.
 */
int32_t hhr_decode_step_host(const hhr_dims* dims, const void* q_host, void* q, const float* R,
                             const float* W, const uint32_t* codes, const void* meta, const void* K,
                             const void* V, int32_t n_valid, int32_t P, int32_t k, float scale,
                             int32_t* page_idx, int32_t* tok_idx, int32_t* n_sel, float* out,
                             float* out_host, void* workspace, size_t ws_bytes, void* stream);

/* Size of the scratch array hhr_decode_step_noalloc uses (4 MiB). */
#define HHR_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * hhr_decode_step without a caller workspace.  The paper has no counterpart:
 * this is a convenience for callers that cannot allocate device memory --
 * for example code whose device memory is fully managed by another
 * framework's allocator it cannot reach, or a host program that is not
 * allowed to allocate after start-up.  The scratch lives in a fixed array of
 * HHR_NOALLOC_SCRATCH_BYTES inside the library; every device that loads the
 * library holds that array until the process exits.
 *   - Arguments and results are those of hhr_decode_step, minus the
 *     workspace; the caller still passes every input and output buffer.
 *   - Sizes whose workspace (hhr_workspace_size) exceeds
 *     HHR_NOALLOC_SCRATCH_BYTES return HHR_ERR_UNSUPPORTED; nothing is
 *     enqueued.  Other argument errors are reported as hhr_decode_step does.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   - The call allocates nothing.  It checks every argument first (a rejected
 *     call enqueues nothing and leaves the array alone), then enqueues a
 *     memset of the array's per-unit counters and the decode kernel.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents: calls that may overlap on the GPU (different streams without
 *     ordering) race and give undefined results.
 *   - The array's status word records a bounded-wait timeout of any call
 *     (outputs of that call are unspecified) and keeps it until
 *     hhr_noalloc_read_status reads it.
 */
int32_t hhr_decode_step_noalloc(const hhr_dims* dims, const void* q, const float* R,
                                const float* W, const uint32_t* codes, const void* meta,
                                const void* K, const void* V, int32_t n_valid, int32_t P,
                                int32_t k, float scale, int32_t* page_idx, int32_t* tok_idx,
                                int32_t* n_sel, float* out, void* stream);

/*
 * Status of hhr_decode_step_noalloc on the current device, as
 * hhr_read_status gives it for a workspace: waits for `stream`, returns the
 * scratch array's status word (HHR_OK or HHR_ERR_TIMEOUT) and clears it.
 * Allocates nothing.  The paper has no counterpart.
 */
int32_t hhr_noalloc_read_status(void* stream);

/*
 * Waits for `stream`, returns the workspace status word (HHR_OK or
 * HHR_ERR_TIMEOUT) and clears it.  After HHR_ERR_TIMEOUT the workspace must be
 * zero-filled again before the next call.  Returns HHR_ERR_CUDA if the copy
 * or the wait fails.
 */
int32_t hhr_read_status(void* workspace, void* stream);

/*
 * Test hook for the bounded waits of the real kernels.  No counterpart in the
 * paper: it exercises the kernels' failure path without any fault.  Arms a
 * one-shot, process-wide flag consumed by the next matching call:
 *   where = 1: the next hhr_select / hhr_decode_step waits at its first unit
 *              barrier (after the page bounds) for one CTA arrival more than
 *              the unit has;
 *   where = 2: the same at its second unit barrier (after the Hamming
 *              distances);
 *   where = 3: the next hhr_encode_keys gives its first pipeline stage one
 *              producer arrival too many, so no tile ever reaches the tensor
 *              cores.
 * That call's waits give up after `spin_cycles` clock cycles (clamped to
 * [1000, 2^32]) instead of about a second, record HHR_ERR_TIMEOUT (read it with
 * hhr_read_status for 1 and 2, hhr_encode_status for 3) and return; nothing
 * is left in flight.  After a decode timeout the workspace must be
 * zero-filled again before the next call.  Outputs of the failed call are
 * unspecified.  Returns HHR_ERR_INVALID_ARG for another `where`.  Not for
 * concurrent use.
 */
int32_t hhr_test_arm_timeout(int32_t where, uint64_t spin_cycles);

#ifdef __cplusplus
}
#endif

#endif /* HHR_H_ */
