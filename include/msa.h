/*
 * msa.h - C ABI of the Memory Sparse Attention (MSA) memory-path library for
 * NVIDIA B200 (sm_100a).
 *
 * One MSA layer's memory path, as the "MSA: Memory Sparse Attention" README
 * describes it ("Architecture" and "Inference Pipeline" sections):
 *   1. msa_pool         - document-wise RoPE on K, then chunk-mean pooling of
 *                         K, V and the router keys Kr into the memory bank.
 *   2.+3. msa_route_topk - cosine routing of the query's router projections Qr
 *                         against the bank's pooled router keys (mean over
 *                         router heads, max over query tokens, max over a
 *                         document's chunks), then the top-k documents.
 *   4. msa_gather       - copy the selected documents' pooled K/V chunks.
 *   5. msa_sparse_attn  - GQA softmax attention of the query tokens over
 *                         [selected memory rows ++ causal local KV].
 *   4.+5. msa_sparse_attn_indexed - the same attention with the selected
 *                         chunks read in place from the bank by index (no
 *                         gathered copy).
 *   msa_layer_forward   - steps 2-5 in one call: msa_route_topk, then
 *                         msa_sparse_attn_indexed.
 * msa_interleave_forward runs several such rounds (the pages' Memory
 * Interleave for multi-hop questions).
 * Beyond the forward path: the backward of steps 5, 4 and 2
 * (msa_sparse_attn_backward, msa_gather_backward, msa_route_backward), the sum
 * of the selected documents' recurrent states that the linear (DGA) layers
 * take as their initial state (msa_state_gather_sum, from the "MSA x Qwen3.5"
 * model card) and the gated delta rule that starts from it
 * (msa_gated_delta_rule), and a routing entry point that allocates nothing
 * (msa_route_topk_noalloc).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.  Every tensor argument is a DEVICE pointer (to memory the caller
 *   allocated and owns) unless its comment says "host".  Tensors are dense,
 *   row-major, innermost dimension last, and 16-byte aligned.  The library
 *   never allocates, frees or synchronises inside these calls.
 * Types.  msa_dtype names the storage type of the float tensors (bf16 or fp32);
 *   every accumulation is fp32.  Offsets are int64, selected indices int32,
 *   scores and normalisers fp32.
 * Streams.  All device work is enqueued on `stream` (a cudaStream_t; NULL is
 *   the legacy default stream), in call order.
 * Errors.  Arguments are checked on the host before anything is launched; a
 *   bad argument returns an error and launches nothing.  A failed launch
 *   returns MSA_ERR_CUDA.  Problems only the device can see (an index out of
 *   range, inconsistent offsets, a bounded wait that ran out) are OR-ed as
 *   MSA_FLAG_* bits into *err_flag (an int32 the caller zeroes beforehand and
 *   reads after synchronising; NULL turns the reporting off); the offending
 *   item is skipped and no kernel traps.
 *   No C++ exception crosses this interface.
 * Reading of the pages (they print no formulas): RoPE is the rotate-half form
 *   with angle p * theta^(-2i/d) for the pair (x_i, x_{i+d/2}), p the token's
 *   position inside its document; it is applied to K only.  The last chunk of
 *   a document may be shorter than P and is averaged over its own tokens.
 *   Attention is bottom-right causal on the local rows (query token i sits at
 *   local position Lloc - Tq + i) and unmasked on memory rows; q-head h reads
 *   KV head h / (Hq / Hkv).
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* msa_stream_t; /* the same type as cudaStream_t */

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = -1, /* null pointer, bad size, misaligned pointer */
  MSA_ERR_UNSUPPORTED = -2, /* a shape or dtype the library has no kernel for */
  MSA_ERR_WORKSPACE = -3,   /* workspace missing or smaller than *_workspace_size */
  MSA_ERR_CUDA = -4,        /* a CUDA launch or runtime call failed */
  MSA_ERR_TOO_LARGE = -5,   /* the problem needs more scratch than msa_route_topk_noalloc holds */
} msa_status;

/* Bits of the device-side error flag. */
enum {
  MSA_FLAG_INDEX_OOB = 1, /* a document / chunk / row index outside its tensor */
  MSA_FLAG_OFFSETS = 2,   /* offsets that are not non-decreasing or disagree with P */
  MSA_FLAG_TIMEOUT = 4,   /* a bounded wait on a barrier ran out */
  MSA_FLAG_OVERFLOW = 8,  /* selected rows exceed the Mmax rows of the output */
};

typedef enum { MSA_F32 = 0, MSA_BF16 = 1 } msa_dtype;

/* Text for a status code; never NULL. */
const char* msa_status_string(int status);

/* Library version, "major.minor.patch". */
const char* msa_version(void);

/* Number of CUDA kernels this library has launched in this process so far
 * (memsets and copies are not kernels and are not counted).  For accounting:
 * the difference across a region is the number of library kernels it ran. */
uint64_t msa_kernel_launch_count(void);

/* For tests of the device-side error path only.  Sets how many times the
 * bf16 prefill attention kernel (msa_sparse_attn and the index-driven
 * attention on prefill shapes) polls each barrier wait that paces its
 * pipeline; a negative value restores the default (2^24).  With 0 every such
 * wait expires at once: the kernel then waits (with the default bound) for the
 * copies and tensor-core operations it already issued, frees its tensor
 * memory, raises MSA_FLAG_TIMEOUT in *err_flag and returns; the outputs of
 * that call are undefined and the next call with the default is unaffected.
 * Process-wide; set it only while no other thread launches the library. */
void msa_testing_set_wait_polls(int64_t polls);

/* ------------------------------------------------------------------------
 * RoPE table (host).  Fills host_out[max_len][d/2][2] with (cos, sin) of the
 * angle p * theta^(-2i/d), computed in fp64 by the C library and stored as
 * fp32, for p < max_len and i < d/2.  The caller copies it to the device for
 * msa_pool.  "MSA: Memory Sparse Attention" README, Figure 2 caption
 * (document-wise RoPE); the rotate-half form is this library's reading.
 * Errors: MSA_ERR_INVALID_ARG for d odd or < 2, max_len < 1, theta <= 0, or a
 * NULL host_out.
 * ---------------------------------------------------------------------- */
msa_status msa_rope_table_host(double theta, int d, int max_len, float* host_out);

/* ------------------------------------------------------------------------
 * Chunk offsets (host).  out[0] = 0 and out[j+1] = out[j] + ceil(L_j / P) with
 * L_j = doc_tok_off[j+1] - doc_tok_off[j]: document j owns chunks
 * [out[j], out[j+1]) of the bank.  doc_tok_off and out are HOST arrays of D+1
 * int64.  Errors: MSA_ERR_INVALID_ARG for NULL arrays, D < 0, P < 1 or a
 * decreasing doc_tok_off.
 * ---------------------------------------------------------------------- */
msa_status msa_chunk_offsets_host(const int64_t* doc_tok_off, int64_t D, int P, int64_t* out);

/* ------------------------------------------------------------------------
 * Step 1: offline memory encoding ("Inference Pipeline", stage 1; "Architecture":
 * chunk-mean pooling of K / V / Kr).  For document j (tokens
 * [doc_tok_off[j], doc_tok_off[j+1]), chunks [doc_chunk_off[j], doc_chunk_off[j+1]))
 * and its chunk c covering tokens [s, e) (P tokens; the last chunk of a document
 * may be shorter):
 *   Kbar[c]  = mean over t in [s,e) of RoPE_{t - doc_tok_off[j]}(K[t])
 *   Vbar[c]  = mean V[t],   Krbar[c] = mean Kr[t]   (not rotated)
 *   kr_rnorm[c, h] = 1 / max(||Krbar_stored[c, h]||, 1e-12)   (fp32, optional)
 * The norm is taken from the stored (rounded) Krbar so that routing sees exactly
 * the bank it reads.
 *   K, V     [Ntok, Hkv, d]   dtype dt
 *   Kr       [Ntok, Hr, dr]   dtype dt
 *   doc_tok_off, doc_chunk_off  int64 [D+1], both starting at 0; document j must
 *            own exactly ceil(L_j / P) chunks and doc_chunk_off[D] == C.
 *   rope_cs  fp32 [max_len, d/2, 2] from msa_rope_table_host; every document
 *            must be at most max_len tokens long.
 *   Kbar, Vbar [C, Hkv, d], Krbar [C, Hr, dr] (dtype dt, outputs)
 *   kr_rnorm fp32 [C, Hr] or NULL.
 * To pool a corpus slab by slab, pass each slab's pointers with offsets that
 * are relative to the slab.  Supported: d, dr in {64, 128}; P in [1, 4096].
 * Device flags: MSA_FLAG_OFFSETS for offsets that disagree with P, Ntok or C,
 * MSA_FLAG_INDEX_OOB for a document longer than max_len (its chunks are skipped).
 * ---------------------------------------------------------------------- */
msa_status msa_pool(msa_dtype dt, const void* K, const void* V, const void* Kr,
                    const int64_t* doc_tok_off, const int64_t* doc_chunk_off,
                    int64_t D, int64_t Ntok, int64_t C, int Hkv, int d, int Hr, int dr, int P,
                    const float* rope_cs, int max_len,
                    void* Kbar, void* Vbar, void* Krbar, float* kr_rnorm,
                    int32_t* err_flag, msa_stream_t stream);

/* kr_rnorm[c, h] = 1 / max(||Krbar[c, h]||, 1e-12) for a bank built elsewhere.
 * Krbar [C, Hr, dr] dtype dt; kr_rnorm fp32 [C, Hr].  dr in {64, 128}. */
msa_status msa_bank_rnorm(msa_dtype dt, const void* Krbar, int64_t C, int Hr, int dr,
                          float* kr_rnorm, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * Steps 2 and 3: routing and top-k ("Architecture": cosine similarity,
 * mean-pooled over heads, then token-wise max, then Top-k documents;
 * "Inference Pipeline" stage 2).
 *   s[b, t, c]       = (1/Hr) sum_h cos(Qr[b, t, h], Krbar[c, h])
 *   doc_score[b, j]  = max over chunks c of document j, max over t < Tq, of s
 *   topk_idx[b, :]   = the k documents with the largest doc_score, sorted by
 *                      score descending, equal scores by lower index first.
 *   Qr        [B, Tq, Hr, dr] dtype dt
 *   Krbar     [C, Hr, dr] dtype dt;  kr_rnorm fp32 [C, Hr] (from msa_pool or
 *             msa_bank_rnorm)
 *   doc_chunk_off int64 [D+1] (a document with no chunks scores -inf)
 *   doc_scores fp32 [B, D] or NULL;  topk_idx int32 [B, k];  topk_score fp32
 *             [B, k] or NULL.
 *   ws / ws_bytes  device scratch of at least msa_route_topk_workspace_size();
 *             its contents need no initialisation and are not kept.
 * Supported: dr in {64, 128}, Hr in [1, 8], 1 <= k <= min(D, 256).
 * Device flags: MSA_FLAG_OFFSETS for decreasing offsets or doc_chunk_off[D] != C.
 * ---------------------------------------------------------------------- */
size_t msa_route_topk_workspace_size(int64_t B, int Tq, int Hr, int64_t D, int64_t C, int k);
msa_status msa_route_topk(msa_dtype dt, const void* Qr, int64_t B, int Tq, int Hr, int dr,
                          const void* Krbar, const float* kr_rnorm,
                          const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                          float* doc_scores, int32_t* topk_idx, float* topk_score,
                          void* ws, size_t ws_bytes, int32_t* err_flag, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * msa_route_topk without a caller workspace.  The pages have no counterpart
 * to this entry point: it exists for callers that cannot allocate device
 * memory when they call the library, such as a plugin whose host framework
 * owns every byte of device memory, or a serving loop that must not allocate
 * after start-up because an allocation can stall on the device or fail under
 * memory pressure.
 * It computes exactly what msa_route_topk computes (same arguments, minus
 * ws / ws_bytes) and allocates nothing: its scratch is a fixed array of
 * MSA_NOALLOC_SCRATCH_BYTES in the library's own device memory, which every
 * GPU that loads the library holds until the process exits.
 *   - Arguments are checked first, exactly as msa_route_topk checks them (a
 *     bad argument returns its own error).  Then problems whose
 *     msa_route_topk_workspace_size() exceeds MSA_NOALLOC_SCRATCH_BYTES return
 *     MSA_ERR_TOO_LARGE.  Either way nothing is queued.  That size is, up to
 *     256-byte rounding of each part, 4 (B D + B) + 4 C + 4 B Tq Hr bytes, plus
 *     8 B k ceil(D / 8192) when D > 8192: the per-document keys and counters,
 *     the chunk -> document map, the query norms and the top-k candidates.
 *     So one query over documents of 8 chunks fits up to 465,768 documents
 *     (3.7 million chunks; Hr = 8, Tq = 64, k = 16), and 64 one-token queries
 *     up to 58,018 documents.
 *   - The first call on each device looks the array's device address up (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - Every call shares the one array, which keeps the previous call's
 *     contents (the routine clears what must start at zero itself).  Calls
 *     that overlap on the GPU, e.g. on two streams at once, race on the array
 *     and must not be issued.
 * ---------------------------------------------------------------------- */
#define MSA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
msa_status msa_route_topk_noalloc(msa_dtype dt, const void* Qr, int64_t B, int Tq, int Hr, int dr,
                                  const void* Krbar, const float* kr_rnorm,
                                  const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                                  float* doc_scores, int32_t* topk_idx, float* topk_score,
                                  int32_t* err_flag, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * Step 4: context assembly ("Inference Pipeline" stage 2: load only the
 * selected K̄ / V̄).  For query b, the chunks of documents topk_idx[b, 0..k-1]
 * are copied in rank order (each document's chunks in ascending order) into
 * rows [0, mem_len[b]) of Kmem / Vmem; rows [mem_len[b], Mmax) are set to zero.
 *   topk_idx int32 [B, k];  doc_chunk_off int64 [D+1]
 *   Kbar, Vbar [C, Hkv, d] dtype dt;  Kmem, Vmem [B, Mmax, Hkv, d];  mem_len int32 [B]
 * Host tier ("Inference Pipeline": the pooled K̄ / V̄ may stay in host memory
 * while K̄r stays on the GPU): Kbar and Vbar may be page-locked host memory
 * that the device addresses directly (cudaHostAlloc, or cudaHostRegister with
 * cudaHostRegisterMapped, under unified addressing); only the selected rows
 * then cross the host link.  Pageable host memory returns
 * MSA_ERR_INVALID_ARG.  The same holds for Kbar / Vbar of msa_layer_forward.
 * Device flags: MSA_FLAG_INDEX_OOB for a document index outside [0, D) or a
 * chunk outside [0, C) (that document is skipped), MSA_FLAG_OVERFLOW when the
 * selected chunks exceed Mmax (the rows that do not fit are dropped).
 * ---------------------------------------------------------------------- */
msa_status msa_gather(msa_dtype dt, const int32_t* topk_idx, int64_t B, int k,
                      const int64_t* doc_chunk_off, int64_t D, int64_t C,
                      const void* Kbar, const void* Vbar, int Hkv, int d, int Mmax,
                      void* Kmem, void* Vmem, int32_t* mem_len,
                      int32_t* err_flag, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * Step 5: sparse attention ("MSA x Qwen3.5" card, "Architecture summary": the
 * top-k chunks' K/V concatenated with the local KV in softmax attention).
 * For batch b, q-head h (KV head g = h / (Hq / Hkv)) and query token i at local
 * position pos_i = Lloc - Tq + i, the keys are memory rows [0, mem_len[b]) of
 * Kmem/Vmem (all visible) followed by local rows [0, pos_i] of Kloc/Vloc:
 *   O[b, i, h] = softmax_j(scale * q . k_j) v_j
 *   lse[b, h, i] = log sum_j exp(scale * q . k_j)    (natural log, optional)
 *   Q [B, Tq, Hq, d];  Kloc, Vloc [B, Lloc, Hkv, d];  Kmem, Vmem [B, Mmax, Hkv, d]
 *   mem_len int32 [B] (each in [0, Mmax]);  O [B, Tq, Hq, d];  lse fp32 [B, Hq, Tq] or NULL
 *   scale <= 0 means 1/sqrt(d).
 * Requires Lloc >= Tq >= 1, Hq % Hkv == 0, d in {64, 128}.  Memory rows
 * [mem_len[b], Mmax) are masked out but must hold finite values: the
 * tensor-core kernels multiply them by zero weights and 0 x NaN is NaN
 * (msa_gather leaves zeros there).
 * Device flags: MSA_FLAG_INDEX_OOB when a mem_len is outside [0, Mmax] (that
 * batch row is computed with mem_len clamped into range).
 * Workspace: msa_sparse_attn_workspace_size bytes, 16-byte aligned; for decode
 * shapes (a few query rows per KV head) the size depends on the current
 * device's SM count, so query it with the device that runs the call current
 * (a workspace that is too small returns MSA_ERR_WORKSPACE and launches
 * nothing).
 * ---------------------------------------------------------------------- */
size_t msa_sparse_attn_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int Mmax);
msa_status msa_sparse_attn(msa_dtype dt, const void* Q, const void* Kloc, const void* Vloc,
                           int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d,
                           const void* Kmem, const void* Vmem, const int32_t* mem_len, int Mmax,
                           float scale, void* O, float* lse,
                           void* ws, size_t ws_bytes, int32_t* err_flag, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * Steps 4 and 5 fused: attention over the selected documents' chunks read in
 * place from the bank ("Inference Pipeline" stage 2: load only the selected
 * K̄ / V̄ and concatenate them with the local context; "MSA x Qwen3.5" card,
 * "Architecture summary").  The result is that of msa_gather followed by
 * msa_sparse_attn with the same Mmax: query b's memory rows are the chunks of
 * documents topk_idx[b, 0..k) in rank order (each document's chunks in
 * ascending order), at most Mmax of them (more raise MSA_FLAG_OVERFLOW and
 * the rows past Mmax are dropped), followed by its causal local rows.
 *   Q, Kloc, Vloc, O, lse, scale as in msa_sparse_attn;
 *   topk_idx int32 [B, k];  doc_chunk_off int64 [D+1];
 *   Kbar, Vbar [C, Hkv, d] dtype dt (device memory, or page-locked host memory
 *   as for msa_gather).
 * For bf16, d = 128 and the shapes the tensor-core kernels take (decode: at most
 * 4 query tokens and 16 query rows per KV head; prefill: a GQA group G that
 * divides 128 with at least 8 tokens per block of 128 rows, and at least
 * min(16, 64 / G) query tokens), a
 * small plan kernel cuts every query's selection into runs of at most 8
 * consecutive chunk rows of one document, and the attention kernel loads those
 * runs straight from the bank with TMA.  A run shorter than 8 rows is padded
 * with masked rows, and decode shapes reserve memory tiles for such padding,
 * so the floating-point summation order (not the keys, not the weights) can
 * differ from msa_sparse_attn's; for prefill shapes and documents whose chunk
 * counts are multiples of 8 the two agree bit for bit.  Other shapes, fp32,
 * and banks in host memory gather the rows into the workspace first and run
 * msa_sparse_attn's kernels.
 * Workspace: msa_sparse_attn_indexed_workspace_size bytes, 16-byte aligned;
 * like msa_sparse_attn's, it depends on the current device's SM count for
 * decode shapes.  Its contents need no initialisation and are not kept.
 * Errors as msa_sparse_attn plus MSA_ERR_INVALID_ARG for k < 1, D < 1, C < 0,
 * missing index / offset / bank pointers, or pageable host banks;
 * MSA_ERR_UNSUPPORTED for k > 65535.  Device flags: MSA_FLAG_INDEX_OOB for a
 * document index outside [0, D) or a chunk range outside [0, C) (that
 * document is skipped), MSA_FLAG_OVERFLOW as above.
 * ---------------------------------------------------------------------- */
size_t msa_sparse_attn_indexed_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int k, int Mmax);
msa_status msa_sparse_attn_indexed(msa_dtype dt, const void* Q, const void* Kloc, const void* Vloc,
                                   int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d,
                                   const int32_t* topk_idx, int k, const int64_t* doc_chunk_off, int64_t D,
                                   int64_t C, const void* Kbar, const void* Vbar, int Mmax, float scale,
                                   void* O, float* lse, void* ws, size_t ws_bytes, int32_t* err_flag,
                                   msa_stream_t stream);

/* ------------------------------------------------------------------------
 * Backward of step 5.  MSA is trained end to end through its sparse attention
 * ("MSA: Memory Sparse Attention" README, "Architecture"; Figure 2 caption);
 * the pages print no gradient, so this is the exact derivative of
 * msa_sparse_attn for an upstream gradient dO:
 *   p_ij = exp(scale q_i.k_j - lse_i),  D_i = sum dO_i * O_i
 *   ds_ij = p_ij (dO_i.v_j - D_i)
 *   dQ_i = scale sum_j ds_ij k_j;  dK_j = scale sum_i ds_ij q_i;  dV_j = sum_i p_ij dO_i
 * the sums over i running over the q-heads of the GQA group and the tokens that
 * see key j.  Inputs as in msa_sparse_attn plus the forward's O (dtype dt) and
 * lse (fp32 [B, Hq, Tq], required) and dO (dtype dt, [B, Tq, Hq, d]).  Outputs
 * are fp32 and fully written: dQ [B, Tq, Hq, d]; dKloc, dVloc [B, Lloc, Hkv, d];
 * dKmem, dVmem [B, Mmax, Hkv, d] (rows past mem_len[b] are zero).  The
 * workspace holds D (msa_sparse_attn_backward_workspace_size bytes).  bf16
 * with d = 128 and the forward's tensor-core GQA shapes runs on tcgen05 kernels
 * (S, dP, dQ, dK and dV contractions on the tensor cores, fp32 accumulators in
 * TMEM); fp32 inputs, d = 64 and other shapes run on CUDA-core kernels with
 * fp32 arithmetic.  Device flags as in msa_sparse_attn.
 * ---------------------------------------------------------------------- */
size_t msa_sparse_attn_backward_workspace_size(int64_t B, int Tq, int Hq);
msa_status msa_sparse_attn_backward(msa_dtype dt, const void* Q, const void* Kloc, const void* Vloc,
                                    int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d,
                                    const void* Kmem, const void* Vmem, const int32_t* mem_len, int Mmax,
                                    float scale, const void* O, const float* lse, const void* dO,
                                    float* dQ, float* dKloc, float* dVloc, float* dKmem, float* dVmem,
                                    void* ws, size_t ws_bytes, int32_t* err_flag, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * Backward of step 4: the adjoint of msa_gather.  Every gathered row's
 * gradient (dKmem / dVmem fp32 [B, Mmax, Hkv, d], rows [0, mem_len[b])) is
 * ADDED into its chunk of dKbar / dVbar (fp32 [C, Hkv, d]; the caller zeroes
 * them, or passes earlier gradients to accumulate); a chunk selected by
 * several queries receives the sum.  topk_idx, doc_chunk_off and mem_len are
 * the ones the forward gather used.  Device flags: MSA_FLAG_INDEX_OOB for a
 * document index or chunk range out of range (that document is skipped).
 * ---------------------------------------------------------------------- */
msa_status msa_gather_backward(const int32_t* topk_idx, int64_t B, int k, const int64_t* doc_chunk_off,
                               int64_t D, int64_t C, const float* dKmem, const float* dVmem,
                               const int32_t* mem_len, int Hkv, int d, int Mmax, float* dKbar, float* dVbar,
                               int32_t* err_flag, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * Backward of step 2 for the selected documents.  A document's routing score
 * is the max over its chunks c and the query's tokens t of the head-mean
 * cosine s(t, c) = (1/Hr) sum_h cos(Qr[b, t, h], Krbar[c, h]) ("MSA: Memory
 * Sparse Attention" README, "Architecture"); the model card's auxiliary
 * routing loss is not defined on the pages, so its gradient with respect to
 * each selected document's score, d_score (fp32 [B, k], laid out as
 * topk_idx), is the input.  The max passes it to its argmax pair (t*, c*),
 * the first in (chunk, token) order on exact ties, with s computed as
 * msa_route_topk computes it (kr_rnorm for the key norms); then for every
 * router head h, with q = Qr[b, t*, h], k = Krbar[c*, h]:
 *   dQr[b, t*, h]  += d_score / Hr * (k / (|q| |k|) - cos(q, k) q / |q|^2)
 *   dKrbar[c*, h]  += d_score / Hr * (q / (|q| |k|) - cos(q, k) k / |k|^2)
 * (norms floored at 1e-12).  Qr, Krbar, kr_rnorm, doc_chunk_off and topk_idx
 * are the ones the forward routing used (dtype dt; fp32 / int64 / int32).
 * dQr (fp32 [B, Tq, Hr, dr]) and dKrbar (fp32 [C, Hr, dr]) are ADDED to: the
 * caller zeroes them or passes earlier gradients; a token or chunk that wins
 * for several documents or queries receives the sum (fp32 atomics, so the
 * summation order is not fixed).  A document with no chunks gets no
 * gradient.  The workspace holds msa_route_backward_workspace_size(B, Tq, k)
 * bytes.  Errors as msa_route_topk; device flags: MSA_FLAG_INDEX_OOB for a
 * document index or chunk range out of range, or a document with more than
 * 2^31 - 1 (chunk, token) pairs (that document is skipped).
 * ---------------------------------------------------------------------- */
size_t msa_route_backward_workspace_size(int64_t B, int Tq, int k);
msa_status msa_route_backward(msa_dtype dt, const void* Qr, int64_t B, int Tq, int Hr, int dr,
                              const void* Krbar, const float* kr_rnorm,
                              const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                              const int32_t* topk_idx, const float* d_score,
                              float* dQr, float* dKrbar,
                              void* ws, size_t ws_bytes, int32_t* err_flag, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * Steps 2-5 for one layer in one call ("Inference Pipeline" stage 2): route +
 * top-k (msa_route_topk), then attention over the selected documents' chunks,
 * read in place from the bank by index, and the local KV
 * (msa_sparse_attn_indexed).  Arguments as in those two calls; Mmax bounds the
 * memory rows per query (selected chunks past it are dropped and flagged
 * MSA_FLAG_OVERFLOW).  topk_idx is required (it is the layer's routing
 * output); doc_scores, topk_score and lse may be NULL.  The workspace is the
 * two calls' workspaces side by side (sized for fp32 storage, so it also
 * covers bf16).
 * ---------------------------------------------------------------------- */
size_t msa_layer_forward_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d,
                                        int Hr, int64_t D, int64_t C, int k, int Mmax);
msa_status msa_layer_forward(msa_dtype dt,
                             const void* Qr, int Hr, int dr,
                             const void* Krbar, const float* kr_rnorm,
                             const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                             const void* Q, const void* Kloc, const void* Vloc,
                             int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d,
                             const void* Kbar, const void* Vbar, int Mmax, float scale,
                             void* O, float* lse, int32_t* topk_idx, float* topk_score,
                             float* doc_scores,
                             void* ws, size_t ws_bytes, int32_t* err_flag, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * Memory Interleave ("MSA: Memory Sparse Attention" README, Figure 3 caption:
 * an optional multi-round interleave after online routing, for multi-hop
 * questions; FAQ "What is Memory Interleave?": multi-round reasoning that
 * jumps across scattered memory segments).  The pages describe it in words
 * only; this library reads it as R rounds of the layer's memory path in which
 * each round retrieves k further documents and reasons over all of them:
 *   round r = 0 .. R-1:
 *     doc_score = routing of Qr_r over the bank (as msa_route_topk)
 *     S_r       = the k best documents not selected in rounds 0 .. r-1
 *                 (documents of earlier rounds score -inf; same order and ties
 *                 as msa_route_topk)
 *     O_r       = attention over the chunks of S_0 ++ S_1 ++ ... ++ S_r (round
 *                 order, then rank order; at most Mmax rows, more raise
 *                 MSA_FLAG_OVERFLOW) ++ the causal local KV
 *                 (msa_sparse_attn_indexed)
 *     Qr_{r+1}  = O_r [B * Tq, Hq * d] x W_route [Hq * d, Hr * dr]  (the
 *                 caller's round-to-round map of the attention output to the
 *                 next router query; fp32 accumulation, stored in dtype dt)
 *   Qr0 [B, Tq, Hr, dr], W_route (required when rounds > 1) dtype dt.
 *   O, lse: the last round's output and log-sum-exp (lse may be NULL).
 *   O_rounds: NULL or [rounds - 1, B, Tq, Hq, d], the earlier rounds' outputs.
 *   Qr_rounds: NULL or [rounds - 1, B, Tq, Hr, dr] (dtype dt), the router
 *   queries of rounds 1 .. rounds-1 as the map stored them.
 *   topk_idx int32 [B, rounds * k] (required): round r's selection in columns
 *   [r k, (r + 1) k);  topk_score fp32 [B, rounds * k] or NULL.
 * Requires rounds * k <= D and B * Tq <= 1,048,560; the rest as
 * msa_layer_forward.  R = 1 is msa_layer_forward.  Workspace:
 * msa_interleave_workspace_size bytes (its contents need no initialisation).
 * ---------------------------------------------------------------------- */
size_t msa_interleave_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int Hr, int dr,
                                     int64_t D, int64_t C, int k, int rounds, int Mmax);
msa_status msa_interleave_forward(msa_dtype dt, const void* Qr0, int Hr, int dr,
                                  const void* Krbar, const float* kr_rnorm,
                                  const int64_t* doc_chunk_off, int64_t D, int64_t C, int k, int rounds,
                                  const void* W_route,
                                  const void* Q, const void* Kloc, const void* Vloc,
                                  int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d,
                                  const void* Kbar, const void* Vbar, int Mmax, float scale,
                                  void* O, float* lse, void* O_rounds, void* Qr_rounds,
                                  int32_t* topk_idx, float* topk_score,
                                  void* ws, size_t ws_bytes, int32_t* err_flag, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * Memory injection of the linear (DGA) layers ("MSA x Qwen3.5" model card,
 * "Architecture summary": the top-k documents' recurrent states are summed
 * into S_ext, the initial state of the query path's gated delta rule).  For
 * query b:
 *   S_ext[b, :] = sum over r < k of states[topk_idx[b, r], :]
 * summed in fp32 in rank order; a document selected twice counts twice.
 *   states [D, S] dtype dt (one recurrent state of S elements per document,
 *   e.g. heads x key dim x value dim);  topk_idx int32 [B, k];  S_ext fp32 [B, S]
 * S must make a state a whole number of 16-byte vectors (S % 8 == 0 for bf16,
 * S % 4 == 0 for fp32), else MSA_ERR_UNSUPPORTED; B <= 65535.  How the states
 * are produced is not part of this library (msa_gated_delta_rule below
 * consumes S_ext).  Device flag: MSA_FLAG_INDEX_OOB for an index outside [0, D); that
 * selection adds nothing.
 * ---------------------------------------------------------------------- */
msa_status msa_state_gather_sum(msa_dtype dt, const void* states, int64_t D, int64_t S,
                                const int32_t* topk_idx, int64_t B, int k, float* S_ext,
                                int32_t* err_flag, msa_stream_t stream);

/* ------------------------------------------------------------------------
 * The linear (DGA) layers' query path ("MSA x Qwen3.5" model card,
 * "Architecture summary": the summed state S_ext of the selected documents is
 * the initial state of the query path's chunked gated delta rule).  The pages
 * do not define the rule; this is the recurrence of Gated DeltaNet (Yang,
 * Kautz and Hatamizadeh, "Gated Delta Networks: Improving Mamba2 with Delta
 * Rule", ICLR 2025), per value head with the state h (key dim x value dim):
 *   h_t = exp(g_t) (I - beta_t k_t k_t^T) h_{t-1} + beta_t k_t v_t^T
 *   o_t = h_t^T (scale q_t)          (scale <= 0 means 1/sqrt(dk))
 * h_0 = h0 (S_ext from msa_state_gather_sum, whose states are laid out
 * [Hv, dk, dv]; NULL means zeros).  Value head h reads key head h / (Hv / Hk).
 *   q, k [B, T, Hk, dk];  v [B, T, Hv, dv];  o [B, T, Hv, dv]   dtype dt
 *   g (log gates, <= 0), beta [B, T, Hv] fp32;  h0, hT fp32 [B, Hv, dk, dv]
 *   (hT, the state after the last token, may be NULL).
 * Keys are used as given (the model normalises them before the rule).
 * Computed in fp32 on the CUDA cores, one CTA per (value head, query):
 * sequences of up to 16 tokens (decode) in the token-by-token form with the
 * state in registers; longer ones chunk by chunk (64 tokens): the within-chunk
 * products, a unit lower-triangular solve for the chunk's new values, then the
 * state update.
 * Supported: dk = dv = 128, Hv % Hk == 0, B <= 65535.  No workspace.
 * ---------------------------------------------------------------------- */
msa_status msa_gated_delta_rule(msa_dtype dt, const void* q, const void* k, const void* v, const float* g,
                                const float* beta, int64_t B, int T, int Hk, int Hv, int dk, int dv,
                                const float* h0, float scale, void* o, float* hT, msa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MSA_H_ */
