/*
 * mmsp.h -- C ABI of libmmsp.so: ring-blockwise causal attention over a
 * zigzag-sharded sequence of interleaved video and text tokens, with all P
 * virtual ranks of the ring computed on one B200 (sm_100a).
 *
 * Method source: "LongVILA Guide: 2M Context Multi-Modal AI Model"
 * (aifetchly blog), sections "Problem" (576 visual tokens per frame,
 * interleaved text), "Multi-Modal Sequence Parallelism (MM-SP) Mechanics"
 * (Ring-SP: each rank holds N/P tokens, K/V blocks travel around the ring in
 * P-1 shifts) and "Implementation" (LongVILAParallelContext ring neighbours;
 * LongVILAMultiModalAttention.forward: (B,S,H,D) layout, scores scaled by
 * 1/sqrt(head_dim), per-step block attention). The log-sum-exp combine, the
 * causal mask, zigzag sharding and GQA head grouping are readings of those
 * passages (the page's sketch sums separately normalised blocks).
 * Extensions on the same path: packed documents with the attention mask
 * reset at each document (section "Critical Operational Best Practices",
 * dynamic sequence packing; mmsp_doc_starts and the doc_start arguments),
 * and the rotary position embedding with base 10^7 fused into the shard
 * gather (three-stage curriculum, Stage 2; mmsp_shard_rope).
 *
 * Conventions for every entry point
 *   - Returns an mmsp_status; MMSP_OK on success. On failure the message of
 *     the calling thread's last error is available from mmsp_last_error().
 *   - All arguments are validated on the host before anything is launched;
 *     a rejected call launches nothing and touches no buffer.
 *   - Device pointers are caller-owned (the library makes no runtime
 *     allocation; its one piece of device memory is the fixed scratch of
 *     mmsp_attn_bwd_noalloc); host pointers are read during the call only.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as
 *     void*; NULL means the legacy default stream). Nothing synchronises.
 *   - bf16 tensors are raw 16-bit bfloat16 words (const void*).
 *   - Token-major layouts: a tensor "[T][H][d]" is row-major with d
 *     contiguous; rank-local tensors are "[P][2C][H][d]" where C = N/(2P)
 *     and rank r's local slot t holds global token
 *         (t < C ? r*C + t : (2P-1-r)*C + (t-C))      (zigzag).
 *   - LSE values are natural logarithms; a row with no visible key has
 *     LSE = -inf and O = 0.
 *   - Device-side waits are bounded; a wait that gives up records a timeout
 *     that mmsp_device_status() reports as MMSP_ETIMEOUT. No kernel traps.
 */
#ifndef MMSP_H
#define MMSP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MMSP_OK = 0,
  MMSP_EINVAL = 1,       /* bad argument (size, alignment, NULL, layout) */
  MMSP_EUNSUPPORTED = 2, /* valid request this build does not implement   */
  MMSP_ECUDA = 3,        /* a CUDA runtime/driver call failed             */
  MMSP_ETIMEOUT = 4      /* a bounded device-side wait gave up            */
} mmsp_status;

/* flags for mmsp_attn_fwd */
#define MMSP_ACCUMULATE 1u /* merge into the running (o_acc, lse) state   */
#define MMSP_FINALIZE 2u   /* also write o_out = bf16(o_acc) (RNE)         */

#define MMSP_MAX_SEGMENTS 4096 /* capacity of the segment table per call */

/*
 * mmsp_shard -- the zigzag shard step: index maps and an optional row permute.
 *
 * Source: "LongVILA Guide", section "MM-SP Mechanics", Ring-SP paragraph
 * (each rank holds N/P tokens), and LongVILAMultiModalAttention.forward's
 * docstring (local length = total / number of ranks). Zigzag (rank r owns
 * chunks r and 2P-1-r of 2P equal chunks) is a reading that balances causal
 * work across ranks.
 *
 *   seg_len, seg_kind  HOST arrays of n_seg entries: the packed sequence as
 *                      segments in order (kind 0 = text, 1 = visual; frames
 *                      are 576-token visual segments). Must sum to N.
 *                      May be NULL (with n_seg = 0) when none of
 *                      modality_local / segid_local / rank_counts is wanted.
 *   N, P               tokens and virtual ranks; N % (2P) == 0, N < 2^31.
 *   local2global       DEVICE int32[N] or NULL: global position of local slot.
 *   global2local       DEVICE int32[N] or NULL: inverse permutation.
 *   modality_local     DEVICE uint8[N] or NULL: kind of each local slot.
 *   segid_local        DEVICE int32[N] or NULL: segment index of each slot.
 *   rank_counts        DEVICE int32[P][2] or NULL: text, visual counts per rank.
 *   src, dst           DEVICE row buffers or both NULL. With inverse == 0:
 *                      dst[l] = src[local2global(l)] (global -> rank-local);
 *                      with inverse != 0: dst[local2global(l)] = src[l].
 *                      Rows are row_bytes long, a multiple of 4 bytes; src and
 *                      dst 16-byte aligned when row_bytes % 16 == 0 (16-byte
 *                      vector path), else 4-byte aligned; no overlap.
 * Bit-exact: pure integer / byte work.
 */
int mmsp_shard(const int32_t* seg_len, const uint8_t* seg_kind, int32_t n_seg,
               int64_t N, int32_t P,
               int32_t* local2global, int32_t* global2local,
               uint8_t* modality_local, int32_t* segid_local, int32_t* rank_counts,
               const void* src, void* dst, int64_t row_bytes, int32_t inverse,
               void* stream);

/*
 * mmsp_shard_frames -- the frame-aligned, modality-balanced shard of the
 * per-token encoder stage, and its re-shard map into the zigzag layout.
 *
 * Source: "LongVILA Guide" (aifetchly), section "Problem" (modality-
 * switching boundaries leave one rank with pure text and another with dense
 * visual patches, and the ranks stall in the collectives). Reading: every
 * frame (visual segment) goes WHOLE to encoder rank floor(P * V_f / V), V_f =
 * visual tokens before it, V = all visual tokens, so every rank holds a
 * contiguous block of frames within one frame of the share V/P; text token
 * number t (text counted alone, T in all) goes to rank floor(P * t / T). The
 * encoder layout concatenates the ranks in order, each rank's frames'
 * tokens (sequence order) then its text tokens (sequence order).
 *
 *   seg_len, seg_kind  HOST table as in mmsp_shard (required, sums to N).
 *   N, P               as mmsp_shard.
 *   global2enc         DEVICE int32[N] or NULL: encoder-layout row of each
 *                      global token.
 *   local2enc          DEVICE int32[N] or NULL: encoder-layout row that
 *                      zigzag rank-local slot l holds, i.e.
 *                      global2enc[local2global[l]]: mmsp_gather_rows with it
 *                      moves the encoder's output into the attention layout
 *                      (scatter: the gradient back).
 *   enc_counts         DEVICE int32[P][2] or NULL: visual, text tokens of
 *                      each encoder rank.
 * Bit-exact integer work.
 */
int mmsp_shard_frames(const int32_t* seg_len, const uint8_t* seg_kind, int32_t n_seg,
                      int64_t N, int32_t P, int32_t* global2enc, int32_t* local2enc,
                      int32_t* enc_counts, void* stream);

/*
 * mmsp_gather_rows -- indexed row copy: dst[i] = src[index[i]] (scatter ==
 * 0) or dst[index[i]] = src[i] (scatter == 1), for i < n_rows; the re-shard
 * between the encoder layout and the zigzag layout (mmsp_shard_frames).
 *
 *   src, dst   DEVICE rows of row_bytes (a multiple of 16), 16-byte
 *              aligned, not overlapping; n_rows rows each.
 *   index      DEVICE int32[n_rows], a permutation of [0, n_rows) for the
 *              scatter. An entry outside [0, n_rows) is skipped and
 *              reported by mmsp_device_status() as MMSP_EINVAL.
 * Bit-exact byte moves; bandwidth-bound.
 */
int mmsp_gather_rows(const void* src, void* dst, const int32_t* index,
                     int64_t n_rows, int64_t row_bytes, int32_t scatter, void* stream);

/*
 * mmsp_shard_rope -- the shard gather of Q or K rows with the rotary
 * position embedding applied on the way (inverse == 0), or the transposed
 * rotation applied while scattering gradient rows back (inverse != 0).
 *
 * Source: "LongVILA Guide" (aifetchly), three-stage curriculum, Stage 2
 * (RoPE base theta raised from 10,000 to 10^7) and section "Distributed
 * Training Configuration" (RoPE base 10,000,000). The pages print no
 * formula; this is the standard rotary embedding: pair (a, b) of each head
 * vector turned by phi_i = pos * theta^(-2i/d), i < d/2:
 *   a' = a cos(phi_i) - b sin(phi_i),  b' = a sin(phi_i) + b cos(phi_i).
 *
 *   src, dst      DEVICE bf16 [N][H][d], 16-byte aligned, not overlapping.
 *                 inverse == 0: dst[l] = R(pos(g)) src[g] with g =
 *                 local2global(l) (global -> rank-local, as mmsp_shard);
 *                 inverse != 0: dst[g] = R(pos(g))^T src[l] (rank-local ->
 *                 global; the gradient of the forward gather).
 *   N, P          as mmsp_shard. H >= 1 heads; d in {8,16,32,64,128,256}.
 *   theta         base, finite and > 1 (10^7 for the long-context stage).
 *   interleaved   0: pairs (i, i + d/2); 1: pairs (2i, 2i + 1).
 *   doc_start     DEVICE int32 [N] (see mmsp_doc_starts) or NULL: pos(g) =
 *                 g - doc_start[g] (positions restart per packed document)
 *                 or g.
 * fp64 angle and range reduction, fp32 rotation, bf16 (RNE) result.
 */
int mmsp_shard_rope(const void* src, void* dst, int64_t N, int32_t P,
                    int32_t H, int32_t d, double theta, int32_t interleaved,
                    const int32_t* doc_start, int32_t inverse, void* stream);

/*
 * mmsp_attn_fwd -- blockwise causal attention of every virtual rank's queries
 * over the K/V blocks it holds at ring steps [step_begin, step_end), merged
 * across steps with the online-softmax (log-sum-exp) combine.
 *
 * Source: "LongVILA Guide", section "Implementation",
 * LongVILAMultiModalAttention.forward (ring loop over ring_size steps; block
 * attention on the current K/V; scores * 1/sqrt(head_dim)) and
 * LongVILAParallelContext (receive from the previous ring rank): at step s,
 * rank r holds the K/V of rank (r - s) mod P.
 *
 *   q                  DEVICE bf16 [P][2C][Hq][d]  rank-local queries
 *   k, v               DEVICE bf16 [P][2C][Hkv][d] rank-local keys/values
 *   N, P, Hq, Hkv, d   N % (2P) == 0; Hq % Hkv == 0; d in {64, 128}.
 *                      Query head h reads kv head floor(h*Hkv/Hq).
 *   scale              softmax scale (1/sqrt(d) for the pages' layer).
 *   causal             1: key j visible to query i iff global j <= global i;
 *                      0: every key visible.
 *   step_begin/end     0 <= begin <= end <= P; (0, P) is the whole ring.
 *   rank_begin/end     0 <= begin < end <= P: the virtual ranks whose queries
 *                      this call computes; (0, P) is every rank. A GPU that
 *                      owns a range of the ring's ranks (the ring split
 *                      across GPUs, "MM-SP Mechanics", Ring-SP paragraph)
 *                      computes its range after gathering every rank's K/V.
 *                      All tensors keep their full [P][2C] shapes: q, o_acc,
 *                      lse and o_out are read/written at the range's rows
 *                      only; k and v are read at every rank's rows.
 *   o_acc              DEVICE fp32 [P][2C][Hq][d]: normalised output over the
 *                      keys seen so far. Read when flags has MMSP_ACCUMULATE,
 *                      written when non-NULL. Required with MMSP_ACCUMULATE.
 *   lse                DEVICE fp32 [P][2C][Hq]: running LSE (natural log).
 *                      Read with MMSP_ACCUMULATE; always written.
 *   o_out              DEVICE bf16 [P][2C][Hq][d]: written (round to nearest
 *                      even) when flags has MMSP_FINALIZE; else may be NULL.
 *   flags              MMSP_ACCUMULATE | MMSP_FINALIZE.
 *   doc_start          DEVICE int32 [N] in GLOBAL order, or NULL: the first
 *                      position of each token's document when several
 *                      documents are packed into one sequence (see
 *                      mmsp_doc_starts). Key j is then visible to query i
 *                      iff doc_start[i] <= j <= i. Needs causal == 1; must
 *                      be non-decreasing with doc_start[i] <= i (not
 *                      checked: other values give unspecified, finite-time
 *                      results). NULL: one document.
 * Without MMSP_ACCUMULATE the state starts empty (LSE -inf, O 0).
 * All pointers 16-byte aligned. fp32 accumulation; tcgen05 tensor cores.
 */
int mmsp_attn_fwd(const void* q, const void* k, const void* v,
                  int64_t N, int32_t P, int32_t Hq, int32_t Hkv, int32_t d,
                  float scale, int32_t causal,
                  int32_t step_begin, int32_t step_end,
                  int32_t rank_begin, int32_t rank_end,
                  float* o_acc, float* lse, void* o_out,
                  uint32_t flags, const int32_t* doc_start, void* stream);

/*
 * mmsp_doc_starts -- doc_start[g] for a packed sequence given as document
 * lengths: the position where the document holding global position g
 * begins.
 *
 * Source: "LongVILA Guide" (aifetchly), section "Critical Operational Best
 * Practices" (dynamic sequence packing: several shorter videos in one long
 * buffer with the attention mask reset between them) and the Stage 3
 * paragraph of the three-stage curriculum (variable-length video segments
 * packed into one long batch). Reading: attention is causal inside each
 * document and nothing crosses a document boundary.
 *
 *   doc_len            HOST int32[n_doc], each >= 1, summing to N;
 *                      1 <= n_doc <= MMSP_MAX_SEGMENTS (ignored when N == 0).
 *   N                  total tokens, 0 <= N < 2^31.
 *   doc_start          DEVICE int32[N] (output), 4-byte aligned.
 * Bit-exact integer work; returns MMSP_EINVAL without launching on bad input.
 */
int mmsp_doc_starts(const int32_t* doc_len, int32_t n_doc, int64_t N,
                    int32_t* doc_start, void* stream);

/*
 * mmsp_lse_merge -- combine two partial attention results over disjoint key
 * sets (the per-step combine of the ring; replaces the page's plain sum of
 * normalised blocks in the ring loop of LongVILAMultiModalAttention.forward):
 *   m = max(la, lb); L = m + ln(e^(la-m) + e^(lb-m));
 *   O = e^(la-L) Oa + e^(lb-L) Ob;   both -inf -> (O, L) = (0, -inf).
 *
 *   o_a, o_b, o_out    DEVICE fp32 [rows][H][d]; o_out may equal o_a or o_b.
 *   lse_a, lse_b, lse_out DEVICE fp32 [rows][H]; lse_out may equal an input.
 *   rows, H, d         d in {4, 8, 16, 32, 64, 128}. o pointers 16-byte
 *                      aligned, lse pointers 4-byte aligned.
 */
int mmsp_lse_merge(const float* o_a, const float* lse_a,
                   const float* o_b, const float* lse_b,
                   float* o_out, float* lse_out,
                   int64_t rows, int32_t H, int32_t d, void* stream);

/*
 * mmsp_ulysses_transpose -- the local sequence <-> head transpose around the
 * Ulysses all-to-all of 2-D MM-SP (P = P_u x P_r).
 *
 * Source: "LongVILA Guide" (aifetchly), section "MM-SP Mechanics"
 * (Ulysses: sequence-sharded (B, N/P, H, D) to head-sharded (B, N, H/P, D)
 * by one all_to_all; the intra-node Ulysses level of MM-SP) and section
 * "Implementation", UlyssesAllToAll (split into P_u contiguous head groups,
 * group j to rank j, received pieces concatenated along the sequence in
 * rank order; the inverse splits the sequence and concatenates the heads;
 * the backward of one is the other).
 *
 *   src, dst     DEVICE buffers, 16-byte aligned, not overlapping; rows of
 *                row_bytes (one head vector; a multiple of 16 bytes).
 *   S            tokens this rank holds (>= 0; 0 is a no-op, pointers
 *                unchecked); H heads, H % P_u == 0;
 *                Hl = H / P_u heads per group.
 *   unpack == 0  pack: src [S][H] -> dst [P_u][S][Hl], dst[j][s][h'] =
 *                src[s][j*Hl + h'] (the send buffer of the forward
 *                all-to-all: block j goes to Ulysses rank j).
 *   unpack == 1  unpack: src [P_u][S][Hl] -> dst [S][H], the inverse (the
 *                receive buffer of the inverse all-to-all, block i from
 *                rank i, back to this rank's tokens with all heads).
 * Bit-exact byte moves; bandwidth-bound.
 */
int mmsp_ulysses_transpose(const void* src, void* dst, int64_t S, int32_t H,
                           int32_t P_u, int64_t row_bytes, int32_t unpack,
                           void* stream);

/*
 * mmsp_attn_bwd -- gradients of the ring attention (whole ring, all P ranks).
 *
 * The pages give only the backward of the all-to-all transpose; this is a
 * reading: the gradient of causal softmax attention, with P_ij = exp(s_ij -
 * LSE_i) recomputed from the saved fp32 LSE and D_i = sum_d dO_i * O_i:
 *   dV_j = sum_i P_ij dO_i;  dS_ij = P_ij (dO_i . v_j - D_i);
 *   dQ_i = scale sum_j dS_ij k_j;  dK_j = scale sum_i dS_ij q_i;
 * dK and dV sum over the Hq/Hkv query heads of each kv head.
 *
 *   q, k, v, o, dout   DEVICE bf16, rank-local, shapes as in mmsp_attn_fwd.
 *   lse                DEVICE fp32 [P][2C][Hq] from mmsp_attn_fwd (whole ring).
 *   dq                 DEVICE bf16 [P][2C][Hq][d]  (output)
 *   dk, dv             DEVICE bf16 [P][2C][Hkv][d] (output)
 *   dq_acc_opt         DEVICE fp32 [P][2C][Hq][d] or NULL: fp32 dQ output.
 *   workspace          DEVICE scratch of at least mmsp_bwd_workspace_bytes()
 *                      bytes (per-head LSE*log2(e) and D rows, about 8*Hq
 *                      bytes per token), 256-byte aligned; contents need not
 *                      be zeroed. Layout: two arrays (LSE*log2(e), then D,
 *                      the second starting mmsp_bwd_workspace_bytes()/2
 *                      bytes in), each fp32 [P][Hq][2][Cp] with Cp = C
 *                      rounded up to a multiple of 128: rank r's rows are
 *                      one contiguous slab of Hq*2*Cp floats per array.
 *   doc_start          as in mmsp_attn_fwd (the same array the forward used).
 *   d == 128 (MMSP_EUNSUPPORTED otherwise); other constraints as
 *   mmsp_attn_fwd.
 */
int mmsp_attn_bwd(const void* q, const void* k, const void* v,
                  const void* o, const void* dout, const float* lse,
                  int64_t N, int32_t P, int32_t Hq, int32_t Hkv, int32_t d,
                  float scale, int32_t causal,
                  void* dq, void* dk, void* dv, float* dq_acc_opt,
                  void* workspace, size_t workspace_bytes,
                  const int32_t* doc_start, void* stream);

/*
 * The three stages mmsp_attn_bwd runs, in this order, exported for callers
 * that want them separately (to time or overlap them, or to skip dQ):
 *   mmsp_attn_bwd_prepare -- D = rowsum(dO * O) and LSE*log2(e) per head
 *                            into `workspace` (one bandwidth-bound kernel);
 *   mmsp_attn_bwd_dkdv    -- dK, dV: key-owner tcgen05 kernel, one kv head
 *                            x 128 keys per work unit;
 *   mmsp_attn_bwd_dq      -- dQ (bf16, plus fp32 into dq_acc_opt if
 *                            non-NULL): query-owner tcgen05 kernel, one
 *                            query head x 128 rows per work item.
 * dkdv and dq read the prepared workspace and may run in either order. The
 * arguments mean what they mean for mmsp_attn_bwd; each call validates its
 * own and returns MMSP_EINVAL/MMSP_EUNSUPPORTED without launching.
 *
 * rank_begin/rank_end (0 <= begin < end <= P; (0, P) = every rank) select
 * the virtual ranks a stage works for, so that a ring split across GPUs
 * runs each stage on the ranks a GPU owns (tensors keep their full [P][2C]
 * shapes, as in mmsp_attn_fwd):
 *   prepare writes the workspace slabs of ranks [begin, end) from those
 *           ranks' rows of o, dout and lse;
 *   dq      writes dQ of the queries of ranks [begin, end); it reads those
 *           ranks' q, dout and workspace slabs and every rank's k, v;
 *   dkdv    writes dK, dV of the keys of ranks [begin, end); it reads those
 *           ranks' k, v and EVERY rank's q, dout and workspace slabs (every
 *           rank's queries may see the keys), so a split ring exchanges
 *           q, dout and the prepared slabs before this stage.
 */
int mmsp_attn_bwd_prepare(const void* o, const void* dout, const float* lse,
                          int64_t N, int32_t P, int32_t Hq, int32_t d,
                          int32_t rank_begin, int32_t rank_end,
                          void* workspace, size_t workspace_bytes, void* stream);
int mmsp_attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout,
                       int64_t N, int32_t P, int32_t Hq, int32_t Hkv, int32_t d,
                       float scale, int32_t causal, int32_t rank_begin, int32_t rank_end,
                       void* dk, void* dv,
                       const void* workspace, size_t workspace_bytes,
                       const int32_t* doc_start, void* stream);
int mmsp_attn_bwd_dq(const void* q, const void* k, const void* v, const void* dout,
                     int64_t N, int32_t P, int32_t Hq, int32_t Hkv, int32_t d,
                     float scale, int32_t causal, int32_t rank_begin, int32_t rank_end,
                     void* dq, float* dq_acc_opt,
                     const void* workspace, size_t workspace_bytes,
                     const int32_t* doc_start, void* stream);

/* Scratch bytes mmsp_attn_bwd needs for these sizes (0 on invalid sizes). */
size_t mmsp_bwd_workspace_bytes(int64_t N, int32_t P, int32_t Hq, int32_t d);

/* Capacity of the library-owned scratch used by mmsp_attn_bwd_noalloc. */
#define MMSP_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * mmsp_attn_bwd_noalloc -- mmsp_attn_bwd for callers that cannot allocate
 * device memory. (No counterpart on the pages: this is an interface
 * convenience of this library.)
 *
 * Some callers own no allocator of their own or must not use one: code
 * embedded in a host framework whose device memory is all handed out by
 * that framework's pool (a cudaMalloc behind its back breaks its
 * accounting), and latency-bound paths where cudaMalloc/cudaFree, which can
 * synchronise the device, are not acceptable between launches. This entry
 * point takes the same inputs and outputs as mmsp_attn_bwd but no
 * workspace: its scratch (the padded per-head LSE/D rows) lives in one
 * file-scope device array of
 * MMSP_NOALLOC_SCRATCH_BYTES (64 MiB) inside libmmsp.so, which every GPU
 * that loads the library keeps until the process exits.
 *
 *   Arguments as mmsp_attn_bwd, without workspace / workspace_bytes.
 *   Sizes whose mmsp_bwd_workspace_bytes() exceeds the capacity are
 *   rejected with MMSP_EINVAL (nothing launched); for example with Hq = 28
 *   N = 262,144 needs about 59 MB and fits, N = 524,288 does not.
 *   The call looks up the array's device address on the current device
 *   (cudaGetSymbolAddress, with that device current) whenever `stream` is
 *   not being captured, so a device reset between calls is harmless. Under
 *   stream capture it reuses the address found by the last uncaptured call
 *   on that device: make the first call on a device before any stream
 *   capture (a first call under capture is rejected with MMSP_EINVAL).
 *   The call allocates nothing (no cudaMalloc, cudaFree or allocating
 *   library routine). All calls on a device share the one array and it keeps
 *   the previous call's contents; everything the kernels need zeroed is
 *   cleared inside the call. Calls that overlap on the GPU (different
 *   streams, or different host threads on one device) race on the array and
 *   must be serialised by the caller.
 */
int mmsp_attn_bwd_noalloc(const void* q, const void* k, const void* v,
                          const void* o, const void* dout, const float* lse,
                          int64_t N, int32_t P, int32_t Hq, int32_t Hkv, int32_t d,
                          float scale, int32_t causal,
                          void* dq, void* dk, void* dv, float* dq_acc_opt,
                          const int32_t* doc_start, void* stream);

/* Message of the calling thread's last failed call ("" if none). */
const char* mmsp_last_error(void);

/*
 * mmsp_device_status -- synchronise `stream`, then report (and clear) a
 * bounded-wait timeout recorded by any kernel of this library on the current
 * device since the previous call: MMSP_ETIMEOUT if one was recorded,
 * MMSP_ECUDA on a CUDA error, else MMSP_OK.
 */
int mmsp_device_status(void* stream);

/*
 * mmsp_selftest_bounded_wait -- launch one CTA that waits on an mbarrier no
 * one arrives on, using the same bounded wait as the attention kernels, with
 * a cap of max_cycles SM clock cycles; the kernel records a timeout and
 * returns. Used by the tests to show that a wait that cannot finish ends with
 * MMSP_ETIMEOUT from mmsp_device_status() instead of hanging.
 * max_cycles in [1, 2^31].
 */
int mmsp_selftest_bounded_wait(int64_t max_cycles, void* stream);

/* Library version string. */
const char* mmsp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MMSP_H */
