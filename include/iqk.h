/*
 * iqk.h -- C ABI of the B200 (sm_100a) IQ2_KS / IQ2_K routed-expert library.
 *
 * Fused dequantization plus matrix-vector / matrix-matrix products over 2-bit
 * IQ_K-family weights, as defined on the mlx-iqk 0.1.1 project page
 * (PKG-INFO), section "Format":
 *
 *   a 2-bit weight reconstructs as  d * float(scale_index) * values[4*alphabet + code],
 *   every step float32, in that order.
 *
 * Stream format (one tensor [rows, cols] per expert; experts stacked on a
 * leading axis; every stream a separate row-major, k-contiguous plane; cols a
 * multiple of 256):
 *
 *   IQ2_KS  qs  uint32 [E][rows][cols/16]   weight k: word k>>4, bits 2*(k&15)..+1
 *           scl uint32 [E][rows][cols/256]  32-weight sub-block j=k>>5: word j>>3,
 *                                           nibble j&7 = low 4 bits of the index
 *           sch uint8  [E][rows][cols/256]  bit j&7 of byte j>>3 = high bit of the index
 *           sex uint8  [E][rows][cols/256]  bit j&7 of byte j>>3 = alphabet bit
 *           dv  uint16 [E][rows]            fp16 row scale (bit pattern)
 *           scale_index = (low4 | high<<4) - 16, in [-16, 15]
 *           row bytes 2 + 70*cols/256 (2.1875 bits per weight + 16 bits per row)
 *
 *   IQ2_K   qs  uint32 [E][rows][cols/16]   as above
 *           scl uint32 [E][rows][cols/128]  16-weight sub-block j=k>>4: word j>>3,
 *                                           nibble j&7; scale_index = nibble - 8
 *           sex uint16 [E][rows][cols/256]  bit j&15 of halfword j>>4 = alphabet bit
 *           dv  uint16 [E][rows][cols/256]  fp16 scale per 256 weights
 *           row bytes 76*cols/256 (2.375 bits per weight)
 *
 * The page fixes the granularity and content of every stream and that codes
 * are little-endian in uint32 words; the packing of scl/sch/sex inside their
 * words, and the offset-16 reading of the IQ2_KS signed index, are this
 * library's readings (offset-16 mirrors IQ2_K's stated offset-8). The
 * eight-entry value table (entries 0-3 alphabet 0, 4-7 alphabet 1) is not
 * printed on the page; every call takes it as an argument.
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller, unless the
 *     parameter says "host". `values` is a host pointer to 8 floats, copied
 *     into the launch (the caller may reuse it on return).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream). Nothing on these paths allocates, frees or
 *     synchronises; scratch comes from the caller's `workspace`.
 *   - Arguments are validated on the host before any launch; a call that
 *     returns an error has enqueued nothing. Device-resident data (expert
 *     ids) is checked on the device: bad ids are skipped and recorded in the
 *     workspace status word (iqk_moe_status).
 *   - bf16 and fp16 values are passed as their 16-bit patterns (uint16_t).
 *   - Every stream plane's base address must be 16-byte aligned (the planes
 *     are staged into shared memory by TMA and bulk copies); IQK_EINVAL if not.
 *   - Consecutive calls overlap their launches: the decode, GEMV,
 *     switch-linear and floor paths launch their kernels as programmatic
 *     dependents of whatever precedes them on the stream. The first kernel
 *     of every call waits (griddepcontrol.wait) for all earlier work on the
 *     stream before it touches any memory, and only then lets the call's
 *     other kernels launch; those read the call's inputs and the weights as
 *     soon as they start, and write outputs only after their own wait. So
 *     stream order holds as usual: a call may read the previous call's
 *     output, and weights written by earlier work on the stream are seen. A
 *     caller's own kernel launched with programmatic stream serialization
 *     right after one of these calls must likewise wait before touching the
 *     call's outputs; kernels launched without that attribute, copies and
 *     events see the call complete, as always.
 */
#ifndef IQK_H_
#define IQK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  IQK_OK = 0,
  IQK_EINVAL = -1,       /* NULL pointer, bad enum, bad id range, inconsistent shapes */
  IQK_ESHAPE = -2,       /* cols not a positive multiple of 256, rows <= 0, ... */
  IQK_EUNSUPPORTED = -3, /* token count / topk / format combination not supported */
  IQK_ECUDA = -4,        /* a CUDA call failed (see iqk_last_cuda_error) */
  IQK_ETIMEOUT = -5,     /* a bounded device wait expired */
  IQK_EWORKSPACE = -6    /* workspace NULL, misaligned (256 B) or too small */
} iqk_status;

typedef enum { IQK_IQ2_KS = 0, IQK_IQ2_K = 1 } iqk_format;

/* One stacked weight tensor: `experts` matrices of [rows, cols]. */
typedef struct {
  int32_t fmt;          /* iqk_format */
  int32_t experts;      /* >= 1 */
  int32_t rows;         /* out_features, >= 1 */
  int32_t cols;         /* in_features, positive multiple of 256 */
  const uint32_t* qs;   /* [experts][rows][cols/16] */
  const uint32_t* scl;  /* IQ2_KS [E][rows][cols/256]; IQ2_K [E][rows][cols/128] */
  const uint8_t* sch;   /* IQ2_KS [E][rows][cols/256]; must be NULL for IQ2_K */
  const void* sex;      /* IQ2_KS uint8 [E][rows][cols/256]; IQ2_K uint16 [E][rows][cols/256] */
  const uint16_t* dv;   /* IQ2_KS [E][rows]; IQ2_K [E][rows][cols/256] */
  /* Optional (NULL when unused): the scale-slot images of these planes,
   * written by iqk_pack_slots, 16-byte aligned. When set, the decode paths
   * (iqk_gemv, iqk_gemv_static, iqk_moe_decode, iqk_moe_decode_host,
   * iqk_moe_decode_shard, the decode kernel of iqk_switch_linear, iqk_floor)
   * fetch each work item's scales with one bulk copy instead of per-lane
   * copies from the planes; iqk_gemv on a matrix of at least 64 row tiles at
   * up to 4 tokens splits rows of a multiple of four blocks into two-block
   * items, whose scales it copies from the planes. The images must have been
   * packed from these same planes. */
  const uint8_t* slots;
} iqk_weights;

/* Human-readable text of a status code (static storage). */
const char* iqk_strerror(int status);
/* Text of the last CUDA error seen by this library in this thread ("" if none). */
const char* iqk_last_cuda_error(void);
/* Library ABI version: 2 (iqk_weights gained `slots`). */
int iqk_version(void);

/*
 * Stream bytes of one row (all planes), or -1 for a bad format / width.
 * Page: "IQ2_KS rows cost 2 + 70*n/256 bytes, IQ2_K rows cost 76*n/256 bytes".
 */
int64_t iqk_row_bytes(int32_t fmt, int32_t cols);

/*
 * Scale-slot images. Page section "Format" (and its note that each stream is
 * rearranged at build time so that values consumed together are contiguous,
 * changing no reconstructed value and no stored byte): the decode kernels
 * take a weight tensor in items of 16 rows x one reduction slice (a fixed
 * number of 256-weight blocks per row, set by cols), and an item needs the
 * slice's bytes of scl, sch and sex and the rows' dv. iqk_pack_slots copies
 * those bytes, for every (expert, 16-row tile, slice), into one contiguous
 * 16-byte-aligned image, zero past the last row. Only the order of the
 * bytes changes.
 *
 * iqk_slots_bytes: bytes of the images of all experts of w (0 if w is
 *   invalid; its `slots` field is ignored).
 * iqk_pack_slots: writes them to `out` (device, 16-byte aligned, at least
 *   iqk_slots_bytes(w) bytes, owned by the caller) on `stream`; IQK_EINVAL
 *   or IQK_EWORKSPACE (out too small or misaligned) before any launch.
 *   Once the copy is complete on the stream, set w.slots = out.
 */
size_t iqk_slots_bytes(const iqk_weights* w);
int iqk_pack_slots(const iqk_weights* w, uint8_t* out, size_t out_bytes, void* stream);

/*
 * iqk_prefill_a_tile -- inspection: the bf16 A operand that iqk_moe_prefill's
 * producer warps decode into tensor memory (page sections "Format" and
 * "Surface": weights dequantized once per expert into the grouped matmul's
 * operand), for rows [row0, row0 + nrows) of expert `expert` of w, all
 * columns, written in k order to out (device, [nrows][cols] bf16 bits).
 *   IQ2_K:  out = bf16_rn((d * float(scale_index)) * values[4*alphabet + code])
 *           (d changes every 256 weights, so it is folded in per weight);
 *   IQ2_KS: out = bf16_rn(float(scale_index) * values[4*alphabet + code]);
 *           the row scale d is applied to the float32 accumulator in the
 *           GEMM epilogue instead.
 * The decode is the producers' own (same tables and per-chunk routine);
 * only the store target differs. IQK_EINVAL before any launch for bad
 * arguments (rows out of range, nrows < 1, out NULL or not 16-byte aligned).
 */
int iqk_prefill_a_tile(const iqk_weights* w, int32_t expert, int32_t row0, int32_t nrows,
                       const float* values /* host [8] */, uint16_t* out, void* stream);

/*
 * iqk_dequant -- reconstruct expert `expert` of `w` to float32, bit-exact.
 * Defines: the reconstruction formula above (page section "Format").
 * out:    device float32 [rows][cols], row-major, written completely.
 * Each weight is (d * (float)scale_index) * values[4*alphabet + code] with
 * both products rounded to nearest even in float32 (no fused multiply-add,
 * no flush of subnormals), so the result equals the CPU dequantizer's.
 * Errors: IQK_EINVAL (NULL, bad fmt, expert out of range), IQK_ESHAPE.
 */
int iqk_dequant(const iqk_weights* w, int32_t expert, const float* values /* host [8] */,
                float* out, void* stream);

/*
 * iqk_dequant_bf16 -- as iqk_dequant, then rounded to bfloat16 (nearest even):
 * out[r][k] = bf16_rn(w_fp32[r][k]). This is the operand the prefill
 * tensor-core path consumes, exposed so it can be checked bit for bit.
 * out: device uint16 [rows][cols].
 */
int iqk_dequant_bf16(const iqk_weights* w, int32_t expert, const float* values /* host [8] */,
                     uint16_t* out, void* stream);

/*
 * iqk_dequant_floor -- the dequantizer's own deleted-decode floor (page
 * section "Pricing": identical loads, decode removed, an integer accumulator
 * reaching the output). It performs the loads and the stores of iqk_dequant
 * (bf16 == 0) or iqk_dequant_bf16 (bf16 != 0) with the reconstruction
 * replaced by integer folding: for qs word wk of row r (weights 16*wk ..
 * 16*wk+15), with the stream fields that word's weights read,
 *   IQ2_KS: m = qs ^ scl_word ^ sch_byte ^ (sex_byte << 8) ^ (dv << 16)
 *           (scl word, sch byte and sex byte of 256-block wk/16; the row's dv)
 *   IQ2_K:  m = qs ^ scl_word ^ (sex_halfword << 8) ^ (dv << 16)
 *           (scl word wk/8; sex halfword and dv of 256-block wk/16)
 * and writes out[r][16*wk + k] = m ^ k, k < 16 (bf16 == 0; out uint32
 * [rows][cols], the bytes of the float32 result) or out[r][8*wk + k] = m ^ k,
 * k < 8 (bf16 != 0; out uint32 [rows][cols/2], the bytes of the bf16 result).
 * out: device, 16-byte aligned, written completely.
 * Errors: IQK_EINVAL (NULL, bad fmt, expert out of range, misaligned out),
 * IQK_ESHAPE.
 */
int iqk_dequant_floor(const iqk_weights* w, int32_t expert, int32_t bf16, uint32_t* out, void* stream);

/*
 * iqk_gemv -- y[t][o] = sum_k w[o][k] * x[t][k] for one expert, t < T.
 * Defines: the fused decode GEMV of the page's "Surface" section (few
 * token-expert pairs, one pass over the reduction axis).
 * x: device bf16 [T][cols], 16-byte aligned; y: device float32 [T][rows];
 * 1 <= T <= 64. A misaligned x returns IQK_EINVAL.
 * Accuracy: |y - y_exact| <= 2e-3 * sum_k |w[o][k] * x[t][k]| (weights enter the
 * tensor-core reduction as bfloat16 of (scale_index * value) with d applied
 * in float32; float32 accumulation).
 * workspace: >= iqk_gemv_workspace_bytes(T, rows, cols) bytes, 256-B aligned.
 */
size_t iqk_gemv_workspace_bytes(int32_t T, int32_t rows, int32_t cols);
int iqk_gemv(const iqk_weights* w, int32_t expert, const float* values /* host [8] */,
             const uint16_t* x, int32_t T, float* y, void* workspace, size_t ws_bytes,
             void* stream);

/*
 * iqk_switch_linear -- the routed single projection of the page's switch
 * linear (section "Surface": IqkSwitchLinear(member, num_experts, out, in),
 * y = proj(x, indices, sorted_indices=True)):
 *     y[t][j][:] = W_{ids[t][j]} x[t]      (float32, one row per pair)
 * for every (token t, slot j). No routing weight, no combine.
 *   w:   [E][rows][cols]; x: device bf16 [T][cols], 16-byte aligned;
 *   ids: device int32 [T][topk]; y: device float32 [T][topk][rows],
 *        16-byte aligned; 1 <= topk <= 16.
 *   mode 1: the decode-style kernel (T <= 64, T * topk <= 1024): one weight
 *           read per run of at most 8 (or 16) pairs of one expert, shared
 *           by the run's pairs;
 *   mode 2: grouped by expert, tcgen05 grouped GEMM (rows a multiple of 256,
 *           T <= 65536);
 *   mode 0: mode 1 up to IQK_SWITCH_DECODE_MAX_PAIRS pairs, else mode 2 (the
 *           page's switch linear also picks its kernel by pair count; the
 *           crossover is measured on B200 at the routed gate geometry,
 *           2048 x 4096 with 256 experts: mode 1 is faster up to 64 tokens
 *           at top-6, 384 pairs).
 * Accuracy as iqk_gemv. Out-of-range ids give zero rows and set bit 0 of the
 * status word (iqk_moe_status reads it from this workspace too).
 * workspace: >= iqk_switch_linear_workspace_bytes(mode, T, topk, E, rows,
 * cols) bytes (0 means the mode cannot take the shape), 256-byte aligned.
 * Returns IQK_EUNSUPPORTED when the chosen mode cannot take the shape.
 */
#define IQK_SWITCH_DECODE_MAX_PAIRS 384
size_t iqk_switch_linear_workspace_bytes(int32_t mode, int32_t T, int32_t topk, int32_t experts, int32_t rows,
                                         int32_t cols);
int iqk_switch_linear(const iqk_weights* w, const float* values /* host [8] */, const uint16_t* x, int32_t T,
                      const int32_t* ids, int32_t topk, float* y, int32_t mode, void* workspace, size_t ws_bytes,
                      void* stream);

/*
 * iqk_gemv_static -- iqk_gemv without a workspace argument (the pages have no
 * counterpart; this is a convenience of this library). The scratch is a
 * file-scope device array of IQK_GEMV_STATIC_SCRATCH_BYTES (4 MiB) in each
 * device context, so the call allocates nothing; it is for callers that
 * cannot allocate device memory at the call site (a plain C host linking only
 * this library, or a code path that must not enter an allocator).
 * A shape whose scratch (iqk_gemv_workspace_bytes) exceeds the array returns
 * IQK_EWORKSPACE. Every call looks the array's address up in the current
 * device context (cudaGetSymbolAddress). Calls overlapping in time on one
 * device share the array and race: serialise them. Arguments and accuracy as
 * iqk_gemv.
 */
#define IQK_GEMV_STATIC_SCRATCH_BYTES (4u << 20)
int iqk_gemv_static(const iqk_weights* w, int32_t expert, const float* values /* host [8] */,
                    const uint16_t* x, int32_t T, float* y, void* stream);

/*
 * Routed-expert block (gate/up GEMV, SwiGLU, down GEMV, weighted combine).
 * Geometry on the page: 256 experts, six selected, gate and up [2048 x 4096],
 * down [4096 x 2048]; any experts >= 1, hidden and inter multiples of 256.
 *
 *   gate, up: [E][inter][hidden];  down: [E][hidden][inter]  (same E)
 *   x:   device bf16 [T][hidden]
 *   ids: device int32 [T][topk], expert of slot j of token t (0 <= id < E;
 *        a token may list one expert in several slots: each slot is its own
 *        pair, weighted by its own p)
 *   p:   device float32 [T][topk], routing weight of each slot
 *   y:   device bf16 [T][hidden], written completely:
 *        y[t] = bf16_rn( sum_j p[t][j] * down_e( bf16_rn( silu(gate_e x_t) * up_e x_t ) ) )
 *        with silu(g) = g / (1 + exp(-g)), e = ids[t][j].
 *   1 <= topk <= 16.
 *
 * iqk_moe_decode: few tokens (1 <= T <= 64); one weight read per distinct
 *   expert per call, shared by the tokens routed to it (an expert with more
 *   than 8 pairs -- 16 when experts average more than 8 -- is read once per
 *   run of that many).
 * iqk_moe_prefill: many tokens (1 <= T <= 65536); pairs grouped by expert,
 *   weights dequantized once per expert into bfloat16 tensor-core operands.
 *
 * workspace: >= iqk_moe_workspace_bytes(...) bytes, 256-B aligned, owned by
 * the caller, not shared by concurrent calls. mode 0 = decode, 1 = prefill.
 */
size_t iqk_moe_workspace_bytes(int32_t mode, int32_t T, int32_t topk, int32_t experts,
                               int32_t hidden, int32_t inter);
int iqk_moe_decode(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down,
                   const float* values /* host [8] */, const uint16_t* x, int32_t T,
                   const int32_t* ids, const float* p, int32_t topk, uint16_t* y,
                   void* workspace, size_t ws_bytes, void* stream);
int iqk_moe_prefill(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down,
                    const float* values /* host [8] */, const uint16_t* x, int32_t T,
                    const int32_t* ids, const float* p, int32_t topk, uint16_t* y,
                    void* workspace, size_t ws_bytes, void* stream);

/*
 * iqk_moe_decode_host -- iqk_moe_decode with x, ids, p and y in page-locked
 * host memory (cudaHostAlloc, cudaMallocHost or cudaHostRegister; reachable
 * from the device at the same address). The call's kernels move the data
 * themselves: its first kernel reads each input byte once over the host link
 * into the workspace, the others read those copies, and the down kernel
 * writes y to host memory. No copy-engine transfer and no host
 * synchronisation is involved: y is complete once `stream` has passed the
 * call (synchronise the stream, or an event recorded after it, before
 * reading y). The caller must not modify x, ids or p until then. Same
 * arguments, accuracy and results as iqk_moe_decode, bit for bit. x must be
 * 16-byte aligned. Returns IQK_EINVAL where one of the four pointers is not
 * page-locked host memory (cudaPointerGetAttributes reports another type),
 * otherwise as iqk_moe_decode. Workspace as iqk_moe_decode (device memory).
 */
int iqk_moe_decode_host(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down,
                        const float* values /* host [8] */, const uint16_t* x /* host */, int32_t T,
                        const int32_t* ids /* host */, const float* p /* host */, int32_t topk,
                        uint16_t* y /* host */, void* workspace, size_t ws_bytes, void* stream);

/*
 * iqk_moe_workspace_layout -- where a routed-block call (mode 0 decode,
 * mode 1 prefill; iqk_moe_decode_shard uses the decode layout) keeps its
 * intermediates inside the caller's workspace, for inspection: the tests
 * read the SwiGLU output h there to check the gate/up stage on its own.
 * Arguments as iqk_moe_workspace_bytes. Fills *out and returns IQK_OK, or
 * IQK_EINVAL (NULL out, a shape the mode cannot take).
 *   status:  byte offset of the int32 status word (iqk_moe_status);
 *   h:       byte offset of h, bf16 [h_rows][inter]. A row holds
 *            bf16_rn(silu(g) * u) of one (token, slot) pair, its inter
 *            elements slot-transposed inside every 16-element group:
 *            element 16w + i + 4j of the pair's h sits at 16w + 4i + j.
 *   h_order: mode 0: -1, row i is pair i = t*topk + j;
 *            mode 1: byte offset of int32 [T*topk]: row i is pair h_order[i]
 *            (pairs in expert order, ties in pair order, as iqk_moe_route);
 *            rows past the number of pairs with a valid id are unused.
 * The values belong to the last call that completed on the workspace.
 */
typedef struct {
  int64_t status;
  int64_t h;
  int64_t h_order;
  int32_t h_rows;
  int32_t reserved;
} iqk_ws_layout;
int iqk_moe_workspace_layout(int32_t mode, int32_t T, int32_t topk, int32_t experts, int32_t hidden,
                             int32_t inter, iqk_ws_layout* out);

/*
 * iqk_moe_decode_shard -- one rank's part of an expert-parallel
 * iqk_moe_decode (the routed block's experts partitioned over ranks; each
 * rank holds the streams of experts [expert_base, expert_base + E) in
 * gate/up/down, E = their `experts`). Arguments as iqk_moe_decode, with the
 * GLOBAL expert ids in `ids`. Pairs whose id lies outside the rank's window
 * are skipped silently (no status bit: they belong to another rank), so a
 * shard checks no ids. Output:
 *   y_partial: device float32 [T][hidden], written completely:
 *     y_partial[t] = sum over slots j with ids[t][j] in the window of
 *                    p[t][j] * down_e( bf16_rn( silu(gate_e x_t) * up_e x_t ) )
 * The sum of every rank's y_partial (a collective, e.g. an all-reduce over
 * NCCL), rounded with iqk_f32_to_bf16, is the routed block's y; summation
 * order across ranks is the collective's. Workspace as iqk_moe_decode.
 */
int iqk_moe_decode_shard(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down,
                         const float* values /* host [8] */, const uint16_t* x, int32_t T,
                         const int32_t* ids, const float* p, int32_t topk, int32_t expert_base,
                         float* y_partial, void* workspace, size_t ws_bytes, void* stream);

/*
 * iqk_moe_prefill_shard -- one rank's part of an expert-parallel prefill, the
 * prefill counterpart of iqk_moe_decode_shard: the rank holds experts
 * [expert_base, expert_base + E) in gate/up/down; ids are global; pairs
 * outside the window are skipped silently. Output
 *   y_partial: device float32 [T][hidden], 16-byte aligned, written completely:
 *     y_partial[t] = sum over slots j in order with ids[t][j] in the window of
 *                    p[t][j] * down_e( bf16_rn( silu(gate_e x_t) * up_e x_t ) )
 * With topk = 1 and p = 1 every row is one pair's float32 down output, the
 * form an all-to-all dispatch / combine ships back to the pair's token
 * (iqk_moe_combine). Workspace and limits as iqk_moe_prefill.
 */
int iqk_moe_prefill_shard(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down,
                          const float* values /* host [8] */, const uint16_t* x, int32_t T,
                          const int32_t* ids, const float* p, int32_t topk, int32_t expert_base,
                          float* y_partial, void* workspace, size_t ws_bytes, void* stream);

/*
 * iqk_moe_combine -- the routed block's weighted combine on its own:
 *   y[t] = bf16_rn( sum over slots j in order of p[t][j] * rows[t*topk + j] )
 * rows: device float32 [T*topk][hidden] (one pair's down output per row, in
 * pair order), 16-byte aligned; p: device float32 [T][topk]; y: device bf16
 * [T][hidden]; hidden a multiple of 4. The same arithmetic, in the same
 * order, as the combine of iqk_moe_prefill.
 */
int iqk_moe_combine(const float* rows, const float* p, int32_t T, int32_t topk, int32_t hidden, uint16_t* y,
                    void* stream);

/*
 * iqk_f32_to_bf16 -- out[i] = bf16_rn(in[i]) (nearest even) for i < n;
 * device pointers. The last step of an expert-parallel decode.
 */
int iqk_f32_to_bf16(const float* in, uint16_t* out, int64_t n, void* stream);

/*
 * iqk_moe_status -- synchronises `stream`, then reads the status word a
 * decode/prefill/switch call left in `workspace`: IQK_OK; IQK_ETIMEOUT if a
 * bounded device wait expired; IQK_EINVAL if any expert id was outside
 * [0, E) (those pairs were skipped). The first applicable code in that order
 * is returned.
 */
int iqk_moe_status(const void* workspace, void* stream);

/*
 * iqk_moe_route -- the prefill grouping step on its own (for inspection):
 * counts[e] = number of (token, slot) pairs routed to e; offsets[e] =
 * exclusive prefix sum (offsets[E] = number of valid pairs); perm[i] = pair
 * index t*topk + j of the i-th pair in expert order, ties in pair order.
 * counts: device int32 [E]; offsets: device int32 [E+1]; perm: device int32 [T*topk]
 * (entries past offsets[E] are left unwritten when ids are out of range).
 * workspace: >= iqk_route_workspace_bytes(T, topk, E) bytes, 256-B aligned;
 * its first word is the status word read by iqk_moe_status. E <= 50000.
 * Page: prefill "honouring the caller's sort flag so each expert's weights are
 * read once per sorted prefill" (section "Surface").
 */
size_t iqk_route_workspace_bytes(int32_t T, int32_t topk, int32_t experts);
int iqk_moe_route(const int32_t* ids, int32_t T, int32_t topk, int32_t experts, int32_t* counts,
                  int32_t* offsets, int32_t* perm, void* workspace, size_t ws_bytes,
                  void* stream);

/*
 * iqk_floor -- the deleted-decode address floor used for pricing (page section
 * "Pricing": identical loads, decode removed, an integer accumulator reaching
 * the output). For each listed expert it streams every byte of every stream
 * of every row with the same access pattern as the decode kernels and writes
 * out[i][r] = XOR over the row's bytes, byte b of a stream folded into byte
 * (b & 3) of a little-endian word.
 * expert_list: device int32 [n_experts]; out: device uint32 [n_experts][rows].
 */
int iqk_floor(const iqk_weights* w, const int32_t* expert_list, int32_t n_experts, uint32_t* out,
              void* stream);

/*
 * iqk_floor_status -- synchronises `stream`, then reports whether a bounded
 * wait of the last iqk_floor call expired: IQK_OK or IQK_ETIMEOUT (that
 * call's checksums are then incomplete). The flag is process-wide per device
 * and cleared by every iqk_floor call; read it before the next one.
 */
int iqk_floor_status(void* stream);

/*
 * iqk_set_wait_limit_ns -- the bound of the device-side waits of the decode,
 * GEMV, switch-linear (decode mode) and floor kernels launched from now on,
 * in nanoseconds of the GPU's global timer (0 restores the default, 2 s).
 * A wait that runs out sets the call's status to IQK_ETIMEOUT
 * (iqk_moe_status, iqk_floor_status); the kernel then lets its copies in
 * flight land (bounded separately, 2 s) and finishes without further loads,
 * and the call's outputs are incomplete.
 * expire != 0 is a testing hook: warp 0 of every CTA of those kernels then
 * also waits once on a barrier nothing arrives on, so the bound runs out on
 * purpose and the timeout path can be exercised; pass 0 for normal work.
 * Process-wide; not synchronised with launches in flight on other threads.
 */
int iqk_set_wait_limit_ns(uint64_t limit_ns, int32_t expire);

#ifdef __cplusplus
}
#endif

#endif /* IQK_H_ */
