/*
 * fa.h — C ABI of libfa.so: exact attention forward on B200 (sm_100a).
 *
 * The operation (page "FlashAttention (VI)", section "Vấn đề của cơ chế
 * attention tiêu chuẩn", plus the masks of "FlashAttention 在昇腾 NPU 上是怎么
 * 省显存的？…" sections "坑一" (causal) and "坑四" (GQA/MQA)):
 *
 *     S   = scale · Q Kᵀ + mask          (mask: 0 or −inf)
 *     O   = softmax_rows(S) · V
 *     LSE = ln Σ_j exp(S_ij)             (per query row, natural log)
 *
 * computed tile by tile with the online-softmax recurrence of "MCU 上
 * Transformer 模型的 Flash Attention 实现在 256KB SRAM 约束下的分块计算与内存
 * 建模方案", §二 (running row max m, running denominator l, rescaled O,
 * division by l at the end), so the N×N matrix S never reaches memory.
 *
 * Masks. Key j is allowed for query row i when j < L_b (key padding; L_b =
 * key_pad_lens[b] clamped to [0, N], or N when key_pad_lens is NULL) and,
 * with causal != 0, when j <= i. Every query row is computed, including rows
 * i >= L_b. A row with no allowed key gets O = 0 and LSE = −inf.
 *
 * GQA/MQA. Query head hq reads K/V head hq / (Hq / Hk) (contiguous groups).
 *
 * Layouts (all contiguous, row-major, same 16-bit dtype for q, k, v, o):
 *     q, o : [B, Hq, N, d]        k, v : [B, Hk, N, d]
 *     lse  : [B, Hq, N] float32   key_pad_lens : [B] int32
 *
 * Ownership. The caller allocates every buffer (device memory) and owns the
 * stream. The library allocates nothing per call and keeps no pointer after
 * the call returns. o and lse must not overlap q, k, v or each other.
 *
 * Asynchrony and errors. fa_fwd validates its arguments on the host and
 * returns a negative fa_status without launching anything when they are
 * invalid; otherwise it enqueues one kernel on `stream` and returns FA_OK
 * (or FA_ERR_CUDA if the launch itself failed). The kernel never traps: each
 * of its waits is bounded, and a wait that runs out records
 * FA_ERR_DEVICE_TIMEOUT in a per-device status word that
 * fa_get_device_status() reads. Messages for the last host-side error of the
 * calling thread come from fa_last_error_string().
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_FP16 = 0, /* IEEE binary16 inputs and output */
  FA_BF16 = 1  /* bfloat16 inputs and output */
} fa_dtype;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = -1,    /* NULL pointer, bad size, misaligned buffer, non-finite scale */
  FA_ERR_UNSUPPORTED = -2,    /* head dim other than 64 or 128, unknown dtype */
  FA_ERR_CUDA = -3,           /* a CUDA runtime/driver call or the launch failed */
  FA_ERR_DEVICE_TIMEOUT = -4  /* a bounded wait inside the kernel ran out */
} fa_status;

/*
 * fa_fwd — one attention forward pass (the whole hot path, one launch).
 *
 *   q, k, v      device pointers, 16-byte aligned, dtype `dtype`.
 *   o            device pointer [B, Hq, N, d], written.
 *   lse          device pointer [B, Hq, N] float32, written; NULL skips it.
 *   B, Hq, Hk, N batch, query heads, K/V heads, sequence length; all >= 1,
 *                Hq % Hk == 0.
 *   d            head dimension: 64 or 128 (the pages ask for a multiple of
 *                16 and use 64 and 128; other values return
 *                FA_ERR_UNSUPPORTED instead of falling back silently).
 *   scale        finite multiplier of Q Kᵀ (usually 1/sqrt(d)); any sign.
 *   causal       0 or 1.
 *   key_pad_lens device pointer to B int32 valid-key counts, or NULL.
 *                Values are clamped to [0, N] in the kernel.
 *   stream       a cudaStream_t (NULL = legacy default stream).
 *   dtype        FA_FP16 or FA_BF16.
 * Returns FA_OK or a negative fa_status.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int Hq, int Hk, int N, int d, float scale, int causal,
           const int32_t* key_pad_lens, void* stream, int dtype);

/*
 * Split-KV forward (the num_splits setting of the GQA page "深度探索Flash-
 * Attention中GQA性能调优技术解析", section "num_splits参数的场景化配置"): the
 * K/V tiles each pair of Q tiles visits are cut into `num_splits` contiguous
 * chunks processed by separate work units, so a problem with few Q tiles
 * still fills the GPU. Each chunk's result (O normalised by its own
 * denominator and its LSE, fp32) goes to `workspace`; a second kernel on the
 * same stream merges the chunks row by row by log-sum-exp:
 *     m = max_s LSE_s,  w_s = exp(LSE_s − m),
 *     O = Σ_s w_s O_s / Σ_s w_s,  LSE = m + ln Σ_s w_s
 * (a chunk with no allowed key has LSE_s = −inf and weight 0). The result
 * equals fa_fwd's up to fp32 rounding.
 *
 *   num_splits       1..16. With 1 this is fa_fwd (workspace unused, may be NULL).
 *   workspace        device pointer, 256-byte aligned, at least
 *                    fa_splitkv_workspace_bytes(B, Hq, N, d, num_splits) bytes,
 *                    overlapping no other argument. Owned by the caller; its
 *                    contents need no initialisation and are scratch after the
 *                    call. Two calls in flight at once (other streams) need
 *                    two workspaces.
 *   workspace_bytes  size of `workspace`.
 *   other arguments  as for fa_fwd.
 * Returns as fa_fwd: FA_OK after enqueuing both kernels, or a negative
 * fa_status (FA_ERR_INVALID_ARG for a bad split count, a short, misaligned or
 * overlapping workspace) with nothing enqueued.
 */
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int Hq, int Hk, int N, int d, float scale, int causal,
                   const int32_t* key_pad_lens, int num_splits, void* workspace,
                   size_t workspace_bytes, void* stream, int dtype);

/*
 * fa_fwd_bias — fa_fwd with an additive bias on the scaled scores:
 *     S = scale · Q Kᵀ + bias + mask,  O = softmax_rows(S) · V,  LSE = ln Σ_j e^{S_ij}.
 * (The CSDN ops-transformer page, section "第一层，算子融合", lists Bias among
 * the operations fused into the attention kernel; its shape is not given
 * there. The bias is not multiplied by scale; the mask applies after it.)
 *
 *   bias          device pointer, 16-byte aligned, dtype `dtype`, contiguous
 *                 [bias_B, bias_H, N, N]: row i, column j is added to the score
 *                 of query i and key j. Finite values or −inf (which removes
 *                 that key for that query); +inf or NaN give undefined results.
 *   bias_B        1 (shared by every batch) or B.
 *   bias_H        1 (shared by every query head) or Hq.
 *   other arguments as for fa_fwd.
 * N must be a multiple of 8 (each bias row is loaded by TMA, which needs
 * 16-byte row strides); other N return FA_ERR_UNSUPPORTED. The bias must not
 * overlap o or lse. Each launch reads the bias blocks of the visited tiles
 * from HBM once per Q tile: B·Hq·N² elements for a full bias (about half
 * with causal), fewer when it is broadcast and L2 catches the reuse.
 * Returns FA_OK or a negative fa_status, as fa_fwd.
 */
int fa_fwd_bias(const void* q, const void* k, const void* v, const void* bias, int bias_B,
                int bias_H, void* o, float* lse, int B, int Hq, int Hk, int N, int d, float scale,
                int causal, const int32_t* key_pad_lens, void* stream, int dtype);

/*
 * fa_bwd — gradients of fa_fwd for an upstream gradient dout = dL/dO:
 *     P = exp(S − LSE) (S the masked scaled scores, LSE the forward's),
 *     dV = Pᵀ·dO,  dP = dO·Vᵀ,  D = rowsum(dO ⊙ O),  dS = P ⊙ (dP − D),
 *     dQ = scale·dS·K,  dK = scale·dSᵀ·Q
 * (the NPU page "FlashAttention 在昇腾 NPU 上是怎么省显存的？…" says the v2
 * kernel reworks the backward so S and P are not stored; P is rebuilt here
 * from Q, K and LSE). A K/V head shared by G query heads receives the sum of
 * their dK, dV.
 *
 *   q, k, v, o, lse  the forward's inputs, output and LSE (o and lse exactly as
 *                    fa_fwd wrote them), layouts as for fa_fwd.
 *   dout             dL/dO, [B, Hq, N, d], dtype `dtype`.
 *   dq               [B, Hq, N, d] written; dk, dv [B, Hk, N, d] written.
 *   workspace        device pointer, 256-byte aligned, at least
 *                    fa_bwd_workspace_bytes(B, Hq, N, d) bytes: an fp32 dQ
 *                    accumulator and two fp32 per-row vectors. Needs no
 *                    initialisation; scratch after the call; one per call in flight.
 *   other arguments  as for fa_fwd (same B, Hq, Hk, N, d, scale, causal,
 *                    key_pad_lens and dtype as the forward call).
 * Enqueues three kernels on `stream`. dq, dk, dv and the workspace must not
 * overlap any other argument. Returns FA_OK or a negative fa_status as fa_fwd;
 * a device whose dynamic shared memory is not 1 KB aligned reports
 * FA_ERR_UNSUPPORTED through fa_get_device_status().
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hk, int N, int d,
           float scale, int causal, const int32_t* key_pad_lens, void* workspace,
           size_t workspace_bytes, void* stream, int dtype);

/* Workspace bytes fa_bwd needs (0 for invalid arguments). */
size_t fa_bwd_workspace_bytes(int B, int Hq, int N, int d);

/*
 * fa_fwd_fp8 — fa_fwd on E4M3 (8-bit float) inputs with per-tensor descale
 * factors: the decoded inputs are Q = q·q_descale, K = k·k_descale,
 * V = v·v_descale, and O = softmax(scale·QKᵀ + mask)·V is written as bfloat16
 * with LSE in fp32 as fa_fwd. (The GQA page "深度探索Flash-Attention中GQA性能
 * 调优技术解析", section "混合精度训练的内存优化", names FP8 for halving the
 * memory traffic; "FlashAttention (VI)" attributes FP8 to FlashAttention-3.)
 * Q·Kᵀ and P·V run on the tensor core in E4M3 with fp32 accumulation; P is
 * rounded to E4M3 for P·V and the row sums use the same rounded values.
 *
 *   q, k, v          device pointers to E4M3 bytes, layouts [B,H,N,d] as fa_fwd.
 *   q_descale, k_descale, v_descale  finite factors > 0.
 *   o                [B, Hq, N, d] bfloat16, written; lse as fa_fwd.
 *   d                128 only; N a multiple of 16 (V is transposed into the
 *                    workspace and loaded by TMA with N-byte rows); other values
 *                    return FA_ERR_UNSUPPORTED.
 *   workspace        device pointer, 256-byte aligned, at least
 *                    fa_fwd_fp8_workspace_bytes(B, Hk, N, d) bytes (the
 *                    transposed V); scratch after the call; one per call in flight.
 *   other arguments  as for fa_fwd.
 * Enqueues two kernels on `stream`. Returns FA_OK or a negative fa_status.
 */
int fa_fwd_fp8(const void* q, const void* k, const void* v, float q_descale, float k_descale,
               float v_descale, void* o, float* lse, int B, int Hq, int Hk, int N, int d,
               float scale, int causal, const int32_t* key_pad_lens, void* workspace,
               size_t workspace_bytes, void* stream);

/* Workspace bytes fa_fwd_fp8 needs (0 for unsupported arguments). */
size_t fa_fwd_fp8_workspace_bytes(int B, int Hk, int N, int d);

/* Workspace bytes fa_fwd_splitkv needs: B·Hq·N·num_splits·(d + 1) floats,
 * each part rounded up to 256 bytes; 0 for num_splits == 1 and for invalid
 * arguments. */
size_t fa_splitkv_workspace_bytes(int B, int Hq, int N, int d, int num_splits);

/*
 * fa_fwd_splitkv_static — fa_fwd_splitkv with the library's own scratch
 * instead of a caller workspace, so the call allocates no memory at all.
 * (The source pages have no counterpart: this is a calling convention of
 * this library, not a step of the method.)
 *
 * Who needs it: callers that cannot allocate device memory per call and hold
 * no pool to carve a workspace from, e.g. a server that reserved nearly all
 * of HBM up front for weights and KV cache (an allocation there can fail in
 * the middle of a request), or a latency-critical loop (cudaMalloc and
 * cudaFree can synchronise the device and stall every stream), or a plain C
 * caller that would otherwise have to keep a workspace alive across
 * asynchronous calls.
 *
 * Scratch: one file-scope device array of FA_STATIC_SCRATCH_BYTES (32 MiB)
 * per device, created when the library's module loads on that device. A
 * problem whose split-KV workspace, fa_splitkv_workspace_bytes(B, Hq, N, d,
 * num_splits), exceeds it is rejected with FA_ERR_INVALID_ARG and a message
 * naming both sizes; nothing is launched. Nothing in the scratch has to start
 * at zero: every partial result the merge reads is written earlier in the
 * same call.
 *
 * Set-up: the first call on each device (with that device current) looks up
 * the scratch's device address with cudaGetSymbolAddress, which may load the
 * module on that device, and sets the kernel's attributes. Make that first
 * call before any stream capture begins.
 *
 * Races: every call on a device shares that one scratch array. Two calls
 * whose kernels can overlap (different streams, or host threads with no
 * ordering between their streams) race on it and corrupt each other's
 * results. Keep such calls on one stream, or use fa_fwd_splitkv with one
 * workspace per stream.
 *
 * Arguments, results and errors as fa_fwd_splitkv, without the workspace.
 */
#define FA_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
int fa_fwd_splitkv_static(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hk, int N, int d, float scale, int causal,
                          const int32_t* key_pad_lens, int num_splits, void* stream,
                          int dtype);

/*
 * fa_fwd_host — fa_fwd on inputs and outputs in HOST memory, with the PCIe
 * copies overlapped with the attention. The pages' user-level call takes whole
 * Q, K, V tensors and returns O (NPU page "FlashAttention 在昇腾 NPU 上是怎么省
 * 显存的？我花了两天把它搞明白了", usage section: flash_attention(q, k, v,
 * block_size, causal)); this is that call for tensors that live on the host.
 *
 *   q, k, v        PINNED host memory (cudaMallocHost, cudaHostAlloc or
 *                  cudaHostRegister), layouts as for fa_fwd; read by
 *                  asynchronous copies after the call returns.
 *   o              pinned host [B, Hq, N, d], written asynchronously.
 *   lse            pinned host [B, Hq, N] float32, or NULL (then lse_dev NULL).
 *   key_pad_lens   pinned host int32 [B] or NULL (no padding).
 *   q_dev .. lens_dev  device buffers of the same sizes (lens_dev [B] int32,
 *                  only with key_pad_lens), owned by the caller; they hold the
 *                  staged inputs and outputs and must not overlap.
 *   num_chunks     0 (library's choice: about 16 MB of inputs per chunk, at
 *                  most 16) or 1..64 wanted chunks: num_chunks runs of whole
 *                  batches when B >= num_chunks, else every batch cut into
 *                  min(Hk, ceil(num_chunks / B)) runs of K/V heads (with their
 *                  query heads); fa_host_chunk_plan lists them.
 *   stream         the caller's stream; other arguments as for fa_fwd.
 *
 * Per chunk: the copy in (q, k, v slices) on a library copy stream, fa_fwd on
 * the chunk's slices on `stream`, the copy out (o, lse slices) on a second
 * library copy stream, ordered by events, so copies in, kernels and copies
 * out of different chunks overlap. The copy streams wait for the work already
 * on `stream`, and `stream` waits for every copy before returning: once
 * `stream` has been synchronised (or waited on), o and lse hold the result
 * and the host inputs may be rewritten. Not before: until then the host
 * inputs must not be written and the outputs not read.
 *
 * Allocates no device memory. The first call on a device creates the two
 * copy streams (kept for the life of the process); each call creates and
 * releases four events. Errors: FA_ERR_INVALID_ARG for pageable host memory,
 * bad sizes, overlapping device buffers; otherwise as fa_fwd. On an error
 * after copies were enqueued, `stream` is still ordered after them.
 */
int fa_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                int Hk, int N, int d, float scale, int causal, const int32_t* key_pad_lens,
                void* q_dev, void* k_dev, void* v_dev, void* o_dev, float* lse_dev,
                int32_t* lens_dev, int num_chunks, void* stream, int dtype);

/* The chunks fa_fwd_host uses for a shape and num_chunks (0: its default):
 * writes {b0, b1, hk0, hk1} per chunk to out[4 * i ..], at most max_chunks
 * chunks, and returns their count (< 0 on bad arguments). Host only. */
int fa_host_chunk_plan(int B, int Hq, int Hk, int N, int d, int num_chunks, int32_t* out,
                       int max_chunks);

/* Message for the last error returned to the calling thread ("" if none).
 * The string is owned by the library (thread-local storage). */
const char* fa_last_error_string(void);

/* Synchronises the current device, then returns and clears its status word:
 * FA_OK, FA_ERR_DEVICE_TIMEOUT, or FA_ERR_CUDA if reading it failed. */
int fa_get_device_status(void);

/* Bound on each in-kernel wait, in milliseconds (default 4000; 1..600000).
 * Returns FA_OK or FA_ERR_INVALID_ARG. Applies to later launches. */
int fa_set_wait_timeout_ms(int ms);

/* ---- schedule introspection (host only; no GPU needed) ------------------
 * The kernel splits the query side into work units of two 128-row Q tiles
 * that share one K/V head: the tiles of one (b, hk) are enumerated by
 * (m-block, query head in the group) and paired in that order. Causal
 * problems list units heaviest first (largest m-block first); each CTA of a
 * persistent grid takes units in a serpentine order. */

/* Number of work units for a problem shape; < 0 on bad arguments. */
int fa_num_units(int B, int Hq, int Hk, int N, int causal);

/* Decodes unit u into out[8] = {b, hk, hq0, mblock0, present0, hq1, mblock1,
 * present1}. Returns FA_OK or FA_ERR_INVALID_ARG. */
int fa_unit_info(int B, int Hq, int Hk, int N, int causal, int u, int32_t* out);

/* With split-KV: unit u of a `num_splits` launch, for a batch whose valid key
 * count is key_len, into out[12] = {b, hk, hq0, mblock0, present0, hq1,
 * mblock1, present1, split, j0, n0, n1}: Q tile t visits K/V tiles
 * [j0, n_t) (none when n_t <= j0). Returns FA_OK or FA_ERR_INVALID_ARG. */
int fa_unit_kv_range(int B, int Hq, int Hk, int N, int causal, int num_splits, int u,
                     int key_len, int32_t* out);

/* Unit taken by CTA `cta` of a `grid`-CTA launch on its iteration `it`
 * (may be >= fa_num_units, meaning that CTA is done). */
int fa_unit_for(int cta, int it, int grid);

/* Causal problems whose grid would have fewer than ~12 CTAs on each (b, hk)
 * head at a time order their units by head groups instead: every level of one
 * group, heaviest first, then the next group, so that about 12 CTAs share each
 * head's K/V tiles in L2 (the query heads of the GQA page "深度探索Flash-
 * Attention中GQA性能调优技术解析" read their shared K/V from cache, section
 * PackGQA). fa_unit_groups returns the number of near-equal groups fa_fwd uses
 * at head dimension d = 128 without a bias on a `grid`-CTA launch of a device
 * with `l2_bytes` of L2: 0 (one group, the plain order) for non-causal
 * problems, problems of fewer than eight waves of units, problems with enough
 * CTAs per head, problems whose K and V (4·N·d bytes a head) fit in half of the
 * L2 already and problems where a group's would not; each group holds at least
 * four waves. < 0 on bad arguments. fa_unit_kv_range_grouped is
 * fa_unit_kv_range with `groups` such groups (0 gives fa_unit_kv_range's
 * order); the first B·Hk mod groups groups hold one head more than the others.
 * Host only. */
int fa_unit_groups(int B, int Hq, int Hk, int N, int d, int causal, int grid, long long l2_bytes);
/* Unit taken by CTA `cta` of a `grid`-CTA launch on its iteration `it` under
 * that order with `groups` >= 2 groups (causal only): the serpentine walk of
 * fa_unit_for restarts in each group, so every group is dealt out evenly by
 * itself. Returns num_units·num_splits once the CTA is done, < 0 on bad
 * arguments. Host only. */
int fa_unit_for_grouped(int B, int Hq, int Hk, int N, int causal, int num_splits, int groups,
                        int cta, int it, int grid);
int fa_unit_kv_range_grouped(int B, int Hq, int Hk, int N, int causal, int num_splits, int groups,
                             int u, int key_len, int32_t* out);

/* Self test of the bounded wait: launches one thread that waits on an
 * mbarrier nothing arrives at, with a limit of `ms` (1..10000) milliseconds,
 * on the legacy default stream, and synchronises. Returns FA_OK when the wait
 * gave up as designed (FA_ERR_DEVICE_TIMEOUT is then left in the status word),
 * FA_ERR_CUDA otherwise. Allocates 8 bytes of device memory for the result. */
int fa_selftest_wait_timeout(int ms);

/* Library version, major*10000 + minor*100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
