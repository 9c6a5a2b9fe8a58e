/*
 * fa_sm100 — exact scaled-dot-product attention for NVIDIA B200 (sm_100a), C ABI.
 *
 * The operation ("Flash Attention V2核心网络算子解析" §二.1, the attention formula;
 * "FlashAttention技术解析：加速GPT训练的核心优化" §2.2, the call's causal / window_size /
 * softmax_scale arguments; "突破大模型训练瓶颈：Flash-Attention编译优化与内存占用解决方案",
 * 滑动窗口注意力, window_size=(left, right)):
 *
 *   S_ij   = scale * q_i . k_j          for keys j visible to query i, else -inf
 *   O_i    = sum_j softmax_j(S_i.) v_j
 *   LSE_i  = ln sum_j exp(S_ij)          (natural log)
 *
 * Visibility: 0 <= j < N, and (win_l == -1 or j >= i - win_l), and
 * (win_r' == -1 or j <= i + win_r'), with win_r' = 0 when causal != 0, else win_r.
 * Window bounds are inclusive; -1 means unbounded. Every query sees at least itself.
 *
 * Layout and types (all calls):
 *   q, k, v, o, dO, dq, dk, dv : contiguous (B, N, H, d) bfloat16 in device memory,
 *                                 base address 16-byte aligned (a TMA requirement).
 *   lse                         : contiguous (B, H, N) float32 in device memory.
 *   d (head dim)                : 64 or 128; anything else returns FA_ERR_UNSUPPORTED.
 *   B, N, H                     : >= 1. scale: any finite float (0 gives uniform weights).
 *
 * Ownership: the caller owns every buffer. The library keeps only per-device caches
 * (SM count, kernel attributes) and one device-side error word per device.
 *
 * Asynchrony and errors: every compute call validates its arguments on the host and
 * returns an fa_status before launching anything; kernels then run asynchronously on
 * `stream` (the legacy default stream when NULL). A launch failure returns FA_ERR_CUDA.
 * Inside the kernels every wait is bounded (about 2 s); a wait that gives up records an
 * error that fa_check() reports as FA_ERR_TIMEOUT, instead of hanging the GPU.
 * Outputs must not overlap inputs (FA_ERR_INVALID_ARG).
 * Thread safety: calls may be made from several host threads.
 */
#ifndef FA_SM100_H
#define FA_SM100_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                      /* same type as cudaStream_t */
typedef struct CUstream_st* fa_stream_t;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size or window, non-finite scale, aliasing */
  FA_ERR_UNSUPPORTED = 2,  /* head dim other than 64 / 128, or no sm_100 device */
  FA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  FA_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up (reported by fa_check) */
  FA_ERR_NO_MEMORY = 5,    /* workspace allocation failed */
  FA_ERR_DEVICE = 6        /* another device-side check failed (reported by fa_check) */
} fa_status;

/*
 * Forward pass. Writes o (B,N,H,d) bf16 and lse (B,H,N) fp32 (natural log).
 * One kernel launch on `stream`.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int N, int H, int d, float scale, int causal, int win_l, int win_r,
           fa_stream_t stream);

/*
 * Forward with an optional ALiBi bias (the call's alibi_slopes, "FlashAttention技术解析：
 * 加速GPT训练的核心优化" §2.2): alibi_slopes is NULL (same as fa_fwd) or a device (B,H)
 * float32 array of slopes m; the score of query i and key j becomes
 * scale * q_i . k_j - m[b*H+h] * |i - j| before the mask and the softmax, and lse is the
 * log-sum-exp of those biased scores. Other arguments and errors as fa_fwd; the slopes must
 * be 4-byte aligned and must not overlap o or lse.
 */
int fa_fwd_ex(const void* q, const void* k, const void* v, const float* alibi_slopes, void* o, float* lse,
              int B, int N, int H, int d, float scale, int causal, int win_l, int win_r,
              fa_stream_t stream);

/*
 * Variable-length batch ("Flash Attention V2核心网络算子解析" §五: variable sequence lengths):
 * B sequences packed along the token axis, sequence b in rows [cu_seqlens[b], cu_seqlens[b+1])
 * of (total,H,d) bf16 tensors q, k, v, o; cu_seqlens is a device (B+1) int32 array with
 * cu_seqlens[0] = 0, non-decreasing, cu_seqlens[B] = total (empty sequences allowed). Each
 * sequence is attended on its own: positions, causal mask and window count from its first
 * token and no token sees another sequence. lse is (H,total) float32. alibi_slopes is NULL or
 * a device (H) float32 array (one slope per head, shared by the sequences). Offsets that break
 * the rules are reported by fa_check() as FA_ERR_DEVICE (every bound the kernels use is
 * clamped into the packed tensor). Other arguments and errors as fa_fwd.
 */
int fa_fwd_varlen(const void* q, const void* k, const void* v, const int* cu_seqlens, const float* alibi_slopes,
                  void* o, float* lse, int B, int total, int H, int d, float scale, int causal, int win_l,
                  int win_r, fa_stream_t stream);

/*
 * FP8 forward ("突破大模型训练瓶颈：Flash-Attention编译优化与内存占用解决方案", 混合精度计算:
 * FP8 inputs with q_descale / k_descale factors). q, k, v are (B,N,H,d) tensors of E4M3
 * codes (OCP 8-bit format: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits), one byte
 * per element, 16-byte aligned; q_descale, k_descale, v_descale are device (B,H) float32
 * arrays: element x of head (b,h) stands for descale[b*H+h] * decode(x). Computes the same
 * O = softmax(scale * Q K^T) V and LSE as fa_fwd on those values, masks as fa_fwd; o is
 * (B,N,H,d) bf16, lse (B,H,N) float32. Q K^T and P V run on the tensor cores in E4M3 with
 * float32 accumulation; P (the unnormalised probabilities, at most 2^8) is rounded to E4M3
 * for P V, the row sums use the unrounded values. d must be 128 (FA_ERR_UNSUPPORTED
 * otherwise). One kernel launch on `stream`; errors as fa_fwd.
 */
int fa_fwd_fp8(const void* q, const void* k, const void* v, const float* q_descale, const float* k_descale,
               const float* v_descale, void* o, float* lse,
               int B, int N, int H, int d, float scale, int causal, int win_l, int win_r,
               fa_stream_t stream);

/*
 * The number of pieces per head fa_decode_paged uses when called with splits = 0, for B
 * sequences of Sq new rows, H heads of dim d and at most max_keys keys per sequence
 * (max_pages * page_size), on the current device: as many as let the H x pieces CTAs run at
 * once (CTAs per SM x SM count / H), at least 1, at most the B * ceil(max_keys / 64) tiles
 * the batch can have and 65535. Negative status on error (-FA_ERR_INVALID_ARG,
 * -FA_ERR_UNSUPPORTED for d other than 64 / 128, Sq > 8 or without an sm_100 device,
 * -FA_ERR_CUDA).
 */
int fa_decode_splits(int B, int Sq, int H, int d, int max_keys);

/*
 * Bytes of device workspace fa_decode_paged needs with `splits` pieces per head: the float32
 * partial outputs (B+splits-1,H,Sq,d) and their log-sum-exps (B+splits-1,H,Sq) of the
 * (sequence, piece) slots, and one int32 arrival counter per (b,h), each region 256-byte
 * aligned; 0 when splits <= 1 (nothing to merge) or for invalid sizes.
 */
size_t fa_decode_workspace_bytes(int B, int Sq, int H, int d, int splits);

/*
 * Attention of the newest query rows against a paged KV cache ("FlashAttention技术解析：加速
 * GPT训练的核心优化" §5, FlashDecoding; "突破大模型训练瓶颈：Flash-Attention编译优化与内存占用
 * 解决方案", Paged KV Cache: the cache in fixed-size pages listed per sequence by a block table).
 *   q            (B,Sq,H,d) bf16: the new rows, 1 <= Sq <= 8; row i of sequence b sits at
 *                position seqlens[b] - Sq + i (the new tokens are already in the cache).
 *   k_cache,
 *   v_cache      (num_pages,page_size,H,d) bf16 page pools; page_size a multiple of 64.
 *   k_new,
 *   v_new        NULL, or (B,Sq,H,d) bf16 rows of the new tokens: written into the caches at
 *                positions seqlens[b] - Sq + i (as flash_attn_with_kvcache updates its cache in
 *                place) before the attention reads them. Both or neither; they, q, o, lse, the
 *                block table and the lengths must not overlap the caches, and a cache row that
 *                receives a new row must not be read by another sequence of the same call (no
 *                page holding a new row is shared, and none appears twice in a block table).
 *   block_table  device (B,max_pages) int32: key j of sequence b is row j % page_size of page
 *                block_table[b*max_pages + j/page_size].
 *   seqlens      device (B) int32: keys held by sequence b (0 <= seqlens[b] <= max_pages*page_size).
 *   o, lse       (B,Sq,H,d) bf16 and (B,H,Sq) float32 natural-log LSE; a row that sees no key
 *                gets O = 0 and LSE = -inf.
 * Masks as fa_fwd, taken at each row's position (causal keeps keys j <= position). d is 64 or
 * 128. `splits` is the number of CTAs per head: each head's visible 64-key tiles, listed
 * sequence after sequence, are cut into that many equal contiguous pieces processed in
 * parallel; a sequence spread over several pieces is merged by log-sum-exp. 0 chooses
 * fa_decode_splits(B,Sq,H,d,max_pages*page_size). With splits > 1 a workspace of
 * fa_decode_workspace_bytes(B,Sq,H,d,splits) bytes (256-byte aligned, any contents) is used;
 * if `workspace` is NULL the call allocates it with cudaMallocAsync/cudaFreeAsync on `stream`.
 * Q K^T and P V run on the tensor cores (bf16 operands, fp32 accumulation; the weights P are
 * rounded to bf16 for the product and O is divided by the sum of the rounded weights; LSE uses
 * the fp32 sum). One launch on `stream` with one piece per head; with more, a small kernel
 * that zeroes the arrival counters and the decode kernel, launched as its programmatic
 * dependent: each CTA writes the new rows that fall in its piece, streams its piece, and the
 * last piece of a
 * sequence to finish merges that sequence's partials. Sequence lengths or page indices that
 * are out of range are not read: the sequence counts as empty (or the page as zeros) and
 * fa_check() returns FA_ERR_DEVICE. Host-visible errors as fa_fwd (splits above 65535 is
 * invalid); Sq > 8 or a page_size that is not a multiple of 64 give FA_ERR_UNSUPPORTED.
 */
int fa_decode_paged(const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                    const int* block_table, const int* seqlens, void* o, float* lse,
                    int B, int Sq, int H, int d, int num_pages, int page_size, int max_pages,
                    float scale, int causal, int win_l, int win_r, int splits,
                    void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Bytes of device workspace fa_bwd needs: a float32 dQ accumulator (B,N,H,d), two
 * float32 (B,H,ceil(N/128)*128) row vectors (-LSE*log2(e) and -D, D = rowsum(dO*O)) and a
 * 256-byte block holding the work counter of the main kernel, each region 256-byte
 * aligned. Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_bytes(int B, int N, int H, int d);

/*
 * Backward pass: given the forward's inputs, its outputs o and lse, and the upstream
 * gradient dO, writes dq, dk, dv (B,N,H,d) bf16 — the gradients of sum(dO * O).
 * `workspace` (device, 256-byte aligned, at least fa_bwd_workspace_bytes) is scratch
 * the call overwrites; if it is NULL the call allocates it with cudaMallocAsync on
 * `stream` and frees it with cudaFreeAsync after its launches.
 * Three launches on `stream`: fa_bwd_preprocess, fa_bwd_main, fa_bwd_dq_convert.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv,
           int B, int N, int H, int d, float scale, int causal, int win_l, int win_r,
           void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Deterministic backward ("FlashAttention技术解析：加速GPT训练的核心优化" §2.2, the call's
 * `deterministic` flag): same arguments, results and workspace as fa_bwd, but dq is
 * accumulated per query tile in a fixed order instead of by additions into a shared fp32
 * accumulator, so repeated calls on the same inputs give bitwise identical dq, dk, dv.
 * Three launches on `stream`: the preprocess, dK/dV, and a dQ kernel that recomputes the
 * scores per query tile (three more matrix products than fa_bwd's dQ path, no atomics).
 */
int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv,
                         int B, int N, int H, int d, float scale, int causal, int win_l, int win_r,
                         void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Backward of fa_fwd_ex: alibi_slopes as there (NULL for none; the slopes are constants of
 * the call and get no gradient), o and lse from fa_fwd_ex with the same slopes;
 * deterministic != 0 selects the algorithm of fa_bwd_deterministic, 0 that of fa_bwd. Other
 * arguments, workspace and errors as fa_bwd.
 */
int fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
              const float* alibi_slopes, void* dq, void* dk, void* dv,
              int B, int N, int H, int d, float scale, int causal, int win_l, int win_r, int deterministic,
              void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Backward of fa_fwd_varlen (same packing, cu_seqlens and alibi_slopes; o and lse from
 * fa_fwd_varlen); deterministic as in fa_bwd_ex. The workspace is that of a single sequence
 * of `total` tokens: fa_bwd_workspace_bytes(1, total, H, d).
 */
int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                  const int* cu_seqlens, const float* alibi_slopes, void* dq, void* dk, void* dv,
                  int B, int total, int H, int d, float scale, int causal, int win_l, int win_r,
                  int deterministic, void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * The three launches of fa_bwd, exposed so that a caller can time or interleave them.
 * Same arguments and rules as fa_bwd, except that `workspace` must be non-NULL and must
 * be the same buffer for the three calls of one backward, issued in this order.
 *   fa_bwd_preprocess : -D = -rowsum(dO * O), -LSE*log2(e), dQ accumulator := 0
 *   fa_bwd_main       : dK, dV (written to dk, dv) and the dQ accumulator
 *   fa_bwd_dq_convert : dq = bf16(dQ accumulator)
 */
int fa_bwd_preprocess(const void* o, const float* lse, const void* dO,
                      int B, int N, int H, int d, void* workspace, size_t workspace_bytes,
                      fa_stream_t stream);
int fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                int B, int N, int H, int d, float scale, int causal, int win_l, int win_r,
                void* workspace, size_t workspace_bytes, fa_stream_t stream);
int fa_bwd_dq_convert(void* dq, int B, int N, int H, int d, void* workspace, size_t workspace_bytes,
                      fa_stream_t stream);

/*
 * Backward pass that allocates nothing (the pages have no counterpart: this is a deployment
 * aid). Same arguments, results and rules as fa_bwd, without the workspace: the scratch it
 * needs lives in a fixed 32 MiB array inside the library's device image, which every GPU
 * that loads the library keeps until the process exits. It is for callers that may not call
 * cudaMalloc / cudaMallocAsync at all — code running under an allocator it does not own,
 * inside a pre-sized memory budget, or on a path where an allocation could fail or stall.
 *   - Problems whose fa_bwd_workspace_bytes() exceeds 32 MiB return FA_ERR_UNSUPPORTED
 *     before anything is launched.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     and caches it; make that first call, on every device, before any stream capture.
 *   - All calls share the one array, and each call rewrites the part it uses (its first
 *     launch zeroes the dQ accumulator and writes the row statistics). Calls that overlap
 *     on the GPU — on two streams, or from two host threads — race on it: serialise them.
 */
int fa_bwd_static_workspace(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dO, void* dq, void* dk, void* dv,
                            int B, int N, int H, int d, float scale, int causal, int win_l, int win_r,
                            fa_stream_t stream);

/*
 * Synchronises `stream` on the current device and reports what the kernels recorded:
 * FA_ERR_TIMEOUT if a device wait gave up, FA_ERR_DEVICE for another device-side check,
 * FA_ERR_CUDA if the synchronisation itself failed, else FA_OK. Clears the record.
 */
int fa_check(fa_stream_t stream);

/* Static, human-readable name of a status code. Never NULL. */
const char* fa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H */
