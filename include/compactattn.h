/*
 * compactattn.h — C ABI of libcompactattn.so: Block-Union KV selection and
 * chunked-prefill attention over the selected blocks of a paged KV cache, for
 * NVIDIA B200 (sm_100a).
 *
 * Method: "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
 * Selection", Abstract.  Per chunk, a 2D block-sparse mask of every query head
 * is used as a KV-selection signal: the mask is OR-ed over the chunk's
 * Q-blocks (Q-block union) and over the query heads that share one KV head
 * (intra-group union), giving one minimal, sorted KV block table per KV head.
 * The chunk's queries then attend to exactly the KV blocks of their group's
 * table, read in place from the paged cache (no KV compaction).
 *
 * Conventions for every call:
 *   - returns CA_OK (0) or a negative CA_ERR_* code; ca_last_error() gives text;
 *   - every pointer argument is a DEVICE pointer owned by the caller, except
 *     where a call says otherwise; the library allocates no device memory;
 *   - every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream); argument errors are reported before anything is
 *     launched, device-side errors through `err_flag`;
 *   - all arrays are C-contiguous with the shapes given below;
 *   - thread safety: calls may come from several host threads; the tensor-map
 *     encoder entry point is resolved once under a lock.
 *
 * Notation: Hq query heads, Hkv KV heads, G = Hq / Hkv heads per group; query
 * head h belongs to group h / G.  B = block = page size in tokens.
 * P = prefix_len, L = chunk_len, nQblk = ceil(L / B), nKblk = ceil((P + L) / B):
 * Q-block qb holds chunk tokens [qb B, qb B + B), KV block kb holds sequence
 * positions [kb B, kb B + B).  P and L need not be multiples of B.
 */
#ifndef COMPACTATTN_H
#define COMPACTATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CA_OK 0
#define CA_ERR_ARG (-1)       /* bad shape, size or null pointer             */
#define CA_ERR_ALIGN (-2)     /* reserved (alignment is no longer required)  */
#define CA_ERR_DTYPE (-3)     /* unsupported dtype code                       */
#define CA_ERR_LAUNCH (-4)    /* a CUDA launch or runtime call failed        */
#define CA_ERR_BOUNDS (-5)    /* device: table entry or page id out of range */
#define CA_ERR_TIMEOUT (-6)   /* device: a bounded pipeline wait ran out     */
#define CA_ERR_WORKSPACE (-7) /* workspace missing or too small              */

/* Bits a kernel ORs into *err_flag (device int32). */
#define CA_FLAG_BOUNDS 1
#define CA_FLAG_TIMEOUT 2

#define CA_DTYPE_BF16 0
#define CA_DTYPE_FP32 1
#define CA_DTYPE_E4M3 2  /* K/V pages of ca_chunk_attention_fp8 (not a Q dtype) */

/*
 * ca_build_tables — Q-block union + intra-group union + compaction
 * ("CompactAttention ...", Abstract: masks become GQA-aware per-group KV
 * block tables, the minimal ones that keep every selected KV block).
 *
 *   mask    uint8 [Hq, nQblk, nKblk]; nonzero = KV block kb selected for
 *           (head h, Q-block qb).  Read as-is: bits above the causal diagonal
 *           are kept (attention's causal rule makes them inert).
 *   tables  int32 [Hkv, nKblk] (out): row g holds the ascending ids of every
 *           block selected by any (h in group g, qb), then -1 padding.
 *   counts  int32 [Hkv] (out): number of valid entries of each row.
 * Limits: 1 <= Hkv <= Hq, Hq % Hkv == 0, nQblk >= 1, 1 <= nKblk <= 65536.
 * The result is bit-exact and deterministic.
 */
int ca_build_tables(const uint8_t* mask, int Hq, int Hkv, int nQblk, int nKblk,
                    int32_t* tables, int32_t* counts, void* stream);

/*
 * ca_build_tables_batched — the same for nb independent masks in one launch
 * (e.g. one mask per layer): masks [nb, Hq, nQblk, nKblk] -> tables
 * [nb, Hkv, nKblk], counts [nb, Hkv].  1 <= nb <= 65535.
 */
int ca_build_tables_batched(const uint8_t* masks, int nb, int Hq, int Hkv, int nQblk,
                            int nKblk, int32_t* tables, int32_t* counts, void* stream);

/*
 * ca_build_tables_bits — the same union and tables from bit-packed masks
 * (one bit per (head, Q-block, KV block) instead of one byte: 8x less to
 * read).  Same method ("CompactAttention ...", Abstract: Q-block union and
 * intra-group union into minimal per-group KV block tables).
 *
 *   mask_bits  uint32 [nb, Hq, nQblk, W], W = ceil(nKblk / 32): bit j (least
 *              significant first) of word w of row (h, qb) selects KV block
 *              32w + j; bits at or past nKblk in the last word are ignored.
 *              4-byte aligned (16-byte alignment with W % 4 == 0 is faster).
 *   tables, counts  as for ca_build_tables_batched.
 * Limits: 1 <= nb <= 65535, Hq % Hkv == 0, nQblk >= 1, 1 <= nKblk <= 65536.
 */
int ca_build_tables_bits(const uint32_t* mask_bits, int nb, int Hq, int Hkv, int nQblk,
                         int nKblk, int32_t* tables, int32_t* counts, void* stream);

/*
 * ca_workspace_size — bytes of device workspace ca_chunk_attention needs for
 * these shapes: bf16 copies of fp32 inputs (dtype == CA_DTYPE_FP32), the
 * schedule and fp32 partial results of the automatic persistent mode
 * (n_splits <= 0), or the fp32 partials of a KV-range split (n_splits > 1).
 * Returns 0 when none is needed, and (size_t)-1 for invalid shapes.
 */
size_t ca_workspace_size(int dtype, int Hq, int Hkv, int head_dim, int block, int chunk_len,
                         int prefix_len, int num_pages, int n_splits);

/*
 * ca_chunk_attention — attention of one prefill chunk over the blocks of its
 * group tables, read in place from a paged KV cache ("CompactAttention ...",
 * Abstract: selected KV blocks accessed in place without KV compaction).
 *
 * For query head h (group g = h / G) and chunk query i at position p = P + i:
 *   keys    J = { j : j / B in tables[g][0 .. counts[g]),  j <= p }
 *   LSE[h,i] = ln sum_{j in J} exp(s_j),  s_j = Q[i,h] . K(j) / sqrt(head_dim)
 *   O[i,h]   = sum_{j in J} exp(s_j - LSE[h,i]) V(j)
 * with K(j) = K_pages[page_table[j / B], g, j % B, :] (V alike).  An empty J
 * gives O = 0 and LSE = -inf.
 *
 *   Q           [L, Hq, d], dtype `dtype` (bf16 or fp32).  The tensor cores
 *               take bf16: an fp32 Q is carried as two bf16 terms
 *               (hi = rn(Q), lo = rn(Q - hi)) so that its rounding does not
 *               shift whole score rows; fp32 K and V are rounded to bf16
 *               (round to nearest even), on the device, into the workspace
 *   K_pages,
 *   V_pages     [num_pages, Hkv, B, d], dtype `dtype`; the chunk's own keys
 *               must already be in their pages, and the rows of the last
 *               block past position P + L - 1 must hold finite values
 *               (ca_append_kv zero-fills them): they are multiplied by zero
 *               weights, and 0 * NaN would poison the row
 *   page_table  int32 [nKblk]: logical block -> physical page
 *   tables,
 *   counts      as written by ca_build_tables for this chunk (ascending rows)
 *   O           [L, Hq, d] (out), dtype `dtype`
 *   LSE         float32 [Hq, L] (out), natural log
 *   workspace   >= ca_workspace_size(...) bytes (may be NULL if that is 0)
 *   n_splits    <= 0: automatic.  bf16: with fewer units (group x 64-token
 *               span x head slice) than SMs, each unit's KV range is split
 *               into floor(SMs / units) pieces (at most 16); otherwise one
 *               CTA per unit, and the units of the last partial wave run as
 *               up to 4 pieces each.  fp32 / E4M3: one CTA per unit when the
 *               units fill the SMs, else a persistent grid of at most one
 *               CTA per SM that splits all units' KV stages evenly.  Pieces
 *               are merged by LSE (needs workspace).  1: one CTA per unit;
 *               k > 1: each unit's KV range split k ways, merged by LSE
 *   err_flag    int32 (device, may be NULL): the kernels OR CA_FLAG_* into it
 *               on an out-of-range table entry / page id (the access is
 *               clamped, results are then undefined) or on a pipeline wait
 *               that exceeded its time limit.  Read it with ca_check().
 * Limits: head_dim in {64, 128}; block in {64, 128}; P >= 0, L >= 1 (any
 * alignment); Hq % Hkv == 0; num_pages >= nKblk.
 */
int ca_chunk_attention(const void* Q, const void* K_pages, const void* V_pages, int dtype,
                       int num_pages, const int32_t* page_table, const int32_t* tables,
                       const int32_t* counts, int Hq, int Hkv, int head_dim, int block,
                       int chunk_len, int prefix_len, void* O, float* LSE, void* workspace,
                       size_t ws_bytes, int n_splits, int32_t* err_flag, void* stream);

/*
 * ca_workspace_size_varlen — bytes of device workspace for
 * ca_chunk_attention_varlen (always > 0: it holds the per-sequence
 * descriptors).  max_kv_len bounds P_s + L_s over the batch (it only sizes
 * KV splits); returns (size_t)-1 for unsupported arguments.
 */
size_t ca_workspace_size_varlen(int dtype, int Hq, int Hkv, int head_dim, int block, int num_seqs,
                                int total_q, int max_kv_len, int num_pages, int n_splits);

/*
 * ca_chunk_attention_varlen — ca_chunk_attention for a batch of sequences,
 * each with its own chunk, prefix, page table and group tables, in one
 * launch (the serving form of chunked prefill: "CompactAttention ...",
 * Abstract, chunked prefill over an accumulated paged KV cache).
 *
 * Sequence s (0 <= s < num_seqs) has L_s = cu_q[s+1] - cu_q[s] chunk tokens
 * at rows [cu_q[s], cu_q[s+1]) of Q / O (columns of LSE) and P_s =
 * prefix_len[s] tokens already cached; its nKblk_s = ceil((P_s + L_s) / B)
 * page-table entries are page_table[cu_pages[s] ...] and its tables
 * [Hkv, nKblk_s] start at tables + Hkv * cu_pages[s] (ca_build_tables output
 * for that sequence); its counts are counts[s * Hkv ...].  Every row follows
 * the single-sequence definition above with the sequence's own P_s, tables
 * and page table.
 *   Q, O        [total_q, Hq, d];  LSE float32 [Hq, total_q]
 *   K_pages,
 *   V_pages     one page pool [num_pages, Hkv, B, d] shared by the batch
 *   cu_q        int32 device [num_seqs + 1], cu_q[0] = 0, cu_q[num_seqs] = total_q
 *   prefix_len  int32 device [num_seqs]
 *   cu_pages    int32 device [num_seqs + 1]: page-table offsets,
 *               cu_pages[s+1] - cu_pages[s] >= nKblk_s
 *   max_kv_len  host bound on P_s + L_s (sizes KV splits)
 *   workspace   >= ca_workspace_size_varlen(...) bytes (never NULL)
 *   n_splits    1: one CTA per unit (sequence, group, 64-token span, head
 *               slice); <= 0: automatic — bf16: when the batch's unit bound
 *               ((ceil(total_q / 64) + num_seqs) x Hkv x head slices) is
 *               below the SM count, each unit's KV range in
 *               floor(SMs / bound) pieces (at most 16, at most
 *               ceil(max_kv_len / 128)), else one CTA per unit; fp32: one
 *               CTA per unit; k > 1: KV range split k ways; pieces merged by
 *               LSE
 * Everything runs on the stream from device arrays (capturable in a CUDA
 * graph).  A sequence whose offsets are inconsistent is skipped (its rows
 * are left unwritten) and CA_FLAG_BOUNDS is set in *err_flag.
 */
int ca_chunk_attention_varlen(const void* Q, const void* K_pages, const void* V_pages, int dtype,
                              int num_pages, int num_seqs, int total_q, const int32_t* cu_q,
                              const int32_t* prefix_len, int max_kv_len,
                              const int32_t* page_table, const int32_t* cu_pages,
                              const int32_t* tables, const int32_t* counts, int Hq, int Hkv,
                              int head_dim, int block, void* O, float* LSE, void* workspace,
                              size_t ws_bytes, int n_splits, int32_t* err_flag, void* stream);

/*
 * ca_chunk_attention_masked — the table builder fused into the attention
 * prologue: ca_chunk_attention for one sequence, reading the chunk's
 * bit-packed masks instead of prebuilt tables ("CompactAttention ...",
 * Abstract: the per-group tables come from a Q-block union and an
 * intra-group union of the masks).  Every CTA ORs its group's G * nQblk mask
 * rows into a bit set in shared memory and ranks it into the ascending table
 * (the same table ca_build_tables_bits writes), then attends exactly as
 * ca_chunk_attention does with that table: the outputs are bit-identical.
 *   mask_bits   uint32 [Hq, nQblk, ceil(nKblk / 32)] (device, 4-byte aligned):
 *               bit j of word w selects KV block 32 w + j; bits past nKblk
 *               are ignored
 *   tables_out, counts_out  optional (may be NULL): [Hkv, nKblk] / [Hkv],
 *               written as ca_build_tables would
 *   workspace   >= ca_workspace_size_masked(...) bytes (may be NULL if 0)
 *   n_splits    <= 0: automatic (KV splits when the units do not fill the
 *               SMs); k >= 1: as for ca_chunk_attention (no persistent mode)
 * Limits: as ca_chunk_attention, and nKblk <= 2048.
 */
size_t ca_workspace_size_masked(int dtype, int Hq, int Hkv, int head_dim, int block,
                                int chunk_len, int prefix_len, int num_pages, int n_splits);
int ca_chunk_attention_masked(const void* Q, const void* K_pages, const void* V_pages, int dtype,
                              int num_pages, const int32_t* page_table, const uint32_t* mask_bits,
                              int Hq, int Hkv, int head_dim, int block, int chunk_len,
                              int prefix_len, int32_t* tables_out, int32_t* counts_out, void* O,
                              float* LSE, void* workspace, size_t ws_bytes, int n_splits,
                              int32_t* err_flag, void* stream);

/*
 * ca_chunk_attention_fp8 — ca_chunk_attention over an FP8 (E4M3) paged KV
 * cache: half the bytes of a bf16 cache per token ("CompactAttention ...",
 * Abstract: selected blocks read in place from the paged cache; the format
 * of the cache is this library's choice).
 *
 * Page format: K_pages / V_pages hold one E4M3 byte per element (1 sign, 4
 * exponent bits with bias 7, 3 mantissa bits; exponent 0 = subnormals; 0x7F
 * / 0xFF are NaN), [num_pages, Hkv, B, d]; K_scale / V_scale float32
 * [num_pages, Hkv] hold one positive, finite scale per (page, KV head):
 * element = decode(byte) * scale.  The result is the single-sequence
 * definition above evaluated on those decoded values.
 *
 * How: the bytes are staged by TMA and widened to f16 (exactly) in shared
 * memory; Q is converted to f16 in the workspace (exact for |Q| in
 * [2^-14, 65504], |Q| must stay below 65504); the MMAs run in f16 with fp32
 * accumulation; the K scale multiplies the scores and the V scale the
 * softmax weights inside the softmax, in fp32 (P is stored as f16, so the
 * per-page scales of one sequence should stay within about 2^10 of each
 * other).
 *   Q       bf16 [L, Hq, d];  O bf16 [L, Hq, d];  LSE float32 [Hq, L]
 *   workspace >= ca_workspace_size_fp8(...) bytes (never 0)
 *   n_splits  <= 0 automatic (KV splits when the units do not fill the SMs),
 *             k >= 1 as for ca_chunk_attention (no persistent grid)
 * Limits: as ca_chunk_attention; one sequence per call.
 */
size_t ca_workspace_size_fp8(int Hq, int Hkv, int head_dim, int block, int chunk_len,
                             int prefix_len, int num_pages, int n_splits);
int ca_chunk_attention_fp8(const void* Q, const uint8_t* K_pages, const uint8_t* V_pages,
                           const float* K_scale, const float* V_scale, int num_pages,
                           const int32_t* page_table, const int32_t* tables,
                           const int32_t* counts, int Hq, int Hkv, int head_dim, int block,
                           int chunk_len, int prefix_len, void* O, float* LSE, void* workspace,
                           size_t ws_bytes, int n_splits, int32_t* err_flag, void* stream);

/*
 * ca_chunk_attention_noalloc — ca_chunk_attention (bf16 inputs) for callers
 * that cannot allocate device memory.  The paper has no counterpart: this is
 * a deployment variant of the same computation.
 *
 * Who needs it: code that runs under an allocator it does not own (e.g. an
 * inference engine that reserves the whole GPU at start-up and forbids
 * cudaMalloc in its forward pass) or a latency-critical loop in which an
 * allocation, and the synchronisation it can imply, is not allowed.  With
 * n_splits > 1 the regular entry point needs caller workspace for the split
 * partials; here they go to a scratch array compiled into the library
 * (ca_noalloc_scratch_bytes() bytes, 32 MiB, which every GPU that loads the
 * library keeps allocated until the process exits).  The caller passes only
 * inputs and outputs; arguments mean what they mean for ca_chunk_attention,
 * with dtype fixed to CA_DTYPE_BF16.
 *
 *   - Shapes whose split partials exceed the scratch size are rejected with
 *     CA_ERR_WORKSPACE (nothing is launched); n_splits <= 0 picks the split
 *     as ca_chunk_attention does.
 *   - The first call on each device looks up the scratch array's device
 *     address (cudaGetSymbolAddress, with that device current) and keeps it
 *     for that device's context; make that first call before any stream
 *     capture.  The address is valid for one context lifetime only: after
 *     cudaDeviceReset (or any new context on the device) the next call looks
 *     it up again, so that call, too, belongs before any capture.
 *   - All calls on a device share the scratch and it keeps the last call's
 *     contents (nothing in it needs to start at zero).  Calls whose kernels
 *     overlap on the GPU race on it: do not run two at once on one device.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
int ca_chunk_attention_noalloc(const void* Q, const void* K_pages, const void* V_pages,
                               int num_pages, const int32_t* page_table, const int32_t* tables,
                               const int32_t* counts, int Hq, int Hkv, int head_dim, int block,
                               int chunk_len, int prefix_len, void* O, float* LSE, int n_splits,
                               int32_t* err_flag, void* stream);

/* Size in bytes of the fixed scratch array ca_chunk_attention_noalloc uses. */
size_t ca_noalloc_scratch_bytes(void);

/*
 * ca_append_kv — write a prefill chunk's new keys and values into the paged
 * KV cache in place, before ca_chunk_attention reads them ("CompactAttention
 * ...", Abstract: chunked prefill over an accumulated, paged KV cache).
 *
 * Token i of the chunk (position p = prefix_len + i) goes to
 * K_pages[page_table[p / B], g, p % B, :] = K_new[i, g, :] (V alike).
 *   K_new, V_new      [chunk_len, Hkv, head_dim], dtype `dtype`
 *   K_pages, V_pages  [num_pages, Hkv, B, head_dim], same dtype (written)
 *   page_table        int32 [ceil((prefix_len + chunk_len) / B)]
 * The rows of the last written block after position prefix_len + chunk_len - 1
 * are set to zero (they are read, with zero weight, by ca_chunk_attention).
 * prefix_len need not be a multiple of B; chunk_len may be 0 (then K_new and
 * V_new may be NULL and nothing is launched).  head_dim * element size must be a
 * multiple of 16 bytes; buffers 16-byte aligned.  A page id out of range sets
 * CA_FLAG_BOUNDS in *err_flag (may be NULL) and that row is skipped.
 */
int ca_append_kv(const void* K_new, const void* V_new, int dtype, void* K_pages, void* V_pages,
                 int num_pages, const int32_t* page_table, int Hkv, int head_dim, int block,
                 int prefix_len, int chunk_len, int32_t* err_flag, void* stream);

/*
 * ca_check — synchronise `stream`, read *err_flag (device int32), clear it,
 * and map it to CA_OK / CA_ERR_BOUNDS / CA_ERR_TIMEOUT.
 */
int ca_check(int32_t* err_flag, void* stream);

/*
 * ca_wait_probe — launch one CTA that waits on a pipeline barrier nobody
 * signals, with a time limit of limit_us microseconds; on expiry it ORs
 * CA_FLAG_TIMEOUT into *err_flag and returns.  Exercises the timeout path of
 * every bounded wait without faulting or hanging the device.
 */
int ca_wait_probe(int32_t* err_flag, int limit_us, void* stream);

/* Copy the last error message of the calling thread into buf (NUL-terminated). */
int ca_last_error(char* buf, size_t n);

/* Library version: major * 10000 + minor * 100 + patch. */
int ca_version(void);

#ifdef __cplusplus
}
#endif
#endif /* COMPACTATTN_H */
