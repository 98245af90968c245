/*
 * fp8gemm.h -- C ABI of the B200 (sm_100a) FP8 block-scaled NT GEMM library.
 *
 * The operation (all three entry points):
 *   C[m, n] = bf16( sum_kb  P_kb[m, n] * sfa[kb][m] * sfb[n / 128][kb] ),
 *   P_kb[m, n] = sum over the 128-wide K block kb of A[m, k] * B[n, k],
 * with A and B in FP8 (e4m3, or e5m2 through the _ex entry points), P_kb computed
 * by the tensor cores and promoted into
 * FP32 accumulators once per K block ("two-level accumulation").
 * Sources:
 *   - "DeepGEMM" how-to (aisharenet.com), "Main functions" 1-3: the dense
 *     gemm_fp8_fp8_bf16_nt and the M-grouped contiguous / masked GEMMs, FP8 in,
 *     BF16 out, only M grouped, experts sharing N and K;
 *   - "DeepGEMM: Efficienza e Precisione..." (turtlesai.it): NT layout only
 *     (LHS not transposed, RHS transposed), fine-grained scaling, LHS scales
 *     laid out for aligned TMA loads, two-level accumulation;
 *   - DeepSeek DeepGEMM news article (senqingzn.com), optimisation and layout
 *     paragraphs: promotion of FP8 tensor-core sums, contiguous layout for
 *     prefill / training, masked layout for decode with unknown expert counts;
 *   - "DeepGEMM" product page (flashmla.org), performance section: the masked
 *     layout is usable under CUDA graphs.
 * The pages leave the scale granularity open; this library fixes it to 1x128
 * for A and 128x128 for B.
 *
 * Layouts (row-major unless stated, all pointers are DEVICE pointers):
 *   A    : e4m3 codes, [M, K] (dense / contiguous) or [G, Mmax, K] (masked).
 *   sfa  : fp32, column-major per K block: element (m, kb) at sfa[kb * ld + m],
 *          ld = fg_sfa_ld(M) (dense / contiguous: M = all rows);
 *          masked: [G][ceil(K/128)][fg_sfa_ld(Mmax)].
 *   B    : e4m3 codes, [N, K] (dense) or [G, N, K] (grouped).
 *   sfb  : fp32, [ceil(N/128), ceil(K/128)] (dense) or [G, ceil(N/128), ceil(K/128)].
 *   C    : bf16, [M, N] (dense / contiguous) or [G, Mmax, N] (masked).
 * Requirements: K % 16 == 0 and N % 8 == 0 (16-byte row strides); A, B, C and
 * sfa 16-byte aligned; sfb 4-byte aligned; K may end in a partial block.
 *
 * Results are deterministic: repeated calls on the same inputs give
 * bit-identical outputs (split-K partials are summed in a fixed order).
 *
 * Ownership: the caller owns every buffer.  The library allocates only in
 * fg_init (a status word, a split-K workspace and its counters), never inside
 * a GEMM call, so calls can be captured into CUDA graphs.  The library's
 * workspace is per device and every GEMM entry point may use it (split tiles of
 * the small-M kernel and of the tiled kernel's last wave), so calls that use it
 * must not run concurrently on different streams of the same device; the _ws
 * entry points take a caller-owned workspace instead (one per stream lets
 * GEMMs run concurrently on several streams).
 *
 * Errors: every entry point returns a status code and never throws.  Argument
 * errors are found on the host before any launch and launch nothing.  A device
 * wait that times out (about two seconds) makes the kernel exit early and sets
 * the device status word, read and cleared by fg_get_device_status().
 */
#ifndef FP8GEMM_H
#define FP8GEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FG_OK = 0,
  FG_ERR_INVALID_ARG = 1,     /* null pointer, negative or inconsistent size */
  FG_ERR_ALIGNMENT = 2,       /* K % 16, N % 8 or a base pointer misaligned */
  FG_ERR_UNSUPPORTED = 3,     /* valid but outside what this build supports (e.g. G > 1024) */
  FG_ERR_NOT_INITIALIZED = 4, /* fg_init was not called for the current device */
  FG_ERR_CUDA = 5,            /* a CUDA runtime / driver call failed */
  FG_ERR_TIMEOUT = 6,         /* a device-side wait ran out; the kernel exited early */
  FG_ERR_DEVICE_CHECK = 7     /* debug build only: a device-side index check failed (an expert index
                                 in m_indices outside [-1, G), a TMA tile coordinate outside its
                                 tensor, a split-K workspace slot or counter out of range); the
                                 kernel finished as a release build would */
} fg_status;

/* FP8 operand formats (the aisharenet.com how-to, "Main functions": the FP8 inputs
 * are E4M3 or E5M2).  The plain entry points take E4M3 for both operands; the _ex
 * variants take each operand's format.  Scales are fp32 in the same layouts for
 * both formats. */
typedef enum {
  FG_E4M3 = 0, /* 1 sign, 4 exponent (bias 7), 3 mantissa bits; largest finite 448 */
  FG_E5M2 = 1  /* 1 sign, 5 exponent (bias 15), 2 mantissa bits; largest finite 57344 */
} fg_fp8_format;

/* Prepare the library on `device` (makes it current): queries the SM count,
 * resolves the tensor-map encoder and allocates the status word, the split-K
 * workspace and counters.  Idempotent.  Call it outside any stream capture. */
fg_status fg_init(int device);

/* Free everything fg_init allocated, on every device it was called for. */
void fg_shutdown(void);

/* Row alignment that each expert's rows must be padded to in the contiguous
 * layout (the block size along M; cf. get_m_alignment_for_contiguous_layout in
 * the aisharenet.com how-to, "Main functions" 2). */
int fg_m_alignment(void);

/* Leading dimension of the column-major A scales for M rows: M rounded up to a
 * multiple of 4, so every K-block column starts on a 16-byte boundary. */
int fg_sfa_ld(int M);

/* Dense C[M,N] = A[M,K] . B[N,K]^T (gemm_fp8_fp8_bf16_nt).  M == 0 is a no-op.
 * stream: a cudaStream_t (NULL = legacy default stream). */
fg_status fp8_gemm_nt(const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                      int M, int N, int K, void* stream);

/* M-grouped contiguous (m_grouped_gemm_fp8_fp8_bf16_nt_contiguous):
 * rows of all experts concatenated along M; m_indices[m] (device, int32) is the
 * expert of row m or -1 for a padding row.  Each expert's rows start at a
 * multiple of fg_m_alignment().  Row m uses B[g] and sfb[g]; padding rows and
 * whole padding blocks are not written.  Indices >= G are treated as -1. */
fg_status fp8_gemm_grouped_contiguous(const void* A, const float* sfa, const void* B, const float* sfb,
                                      void* C, const int* m_indices, int M_total, int G, int N, int K,
                                      void* stream);

/* M-grouped masked (m_grouped_gemm_fp8_fp8_bf16_nt_masked): group g owns rows
 * [0, masked_m[g]) of A[g]; masked_m lives in DEVICE memory and is never read
 * by the host, so the launch has a fixed shape and can be captured in a CUDA
 * graph and replayed with new counts.  Rows at or past masked_m[g] of C[g] are
 * left untouched; counts above Mmax are clamped to Mmax. */
fg_status fp8_gemm_grouped_masked(const void* A, const float* sfa, const void* B, const float* sfb,
                                  void* C, const int* masked_m, int G, int Mmax, int N, int K,
                                  void* stream);

/* The three GEMMs above with an explicit format for A (fmt_a) and for B (fmt_b):
 * FG_E4M3 or FG_E5M2 each, mixed allowed; any other value is FG_ERR_INVALID_ARG.
 * Everything else is as for the plain entry points. */
fg_status fp8_gemm_nt_ex(const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                         int M, int N, int K, int fmt_a, int fmt_b, void* stream);
fg_status fp8_gemm_grouped_contiguous_ex(const void* A, const float* sfa, const void* B, const float* sfb,
                                         void* C, const int* m_indices, int M_total, int G, int N, int K,
                                         int fmt_a, int fmt_b, void* stream);
fg_status fp8_gemm_grouped_masked_ex(const void* A, const float* sfa, const void* B, const float* sfb,
                                     void* C, const int* masked_m, int G, int Mmax, int N, int K,
                                     int fmt_a, int fmt_b, void* stream);

/* Size in bytes of a caller-owned split-K workspace for the current device (it depends on
 * the SM count): two fp32 partial tiles of 128 x 256 per SM, then 65536 int32 counters.
 * 0 if fg_init was not called for the device. */
size_t fg_workspace_bytes(void);

/* Call options (the `flags` argument of the _ws entry points), or-ed together.
 * FG_FLAG_STATIC_B: B and sfb are not written by the kernel that immediately precedes this
 *   call on its stream (weights loaded once and reused, as in inference).  The kernel may
 *   then start loading weight tiles before that kernel has finished (it still waits for it
 *   before touching A, sfa, C or the workspace), which hides the hand-over between
 *   back-to-back launches.  Taken by the small-M kernel (dense M <= 128); the other kernels
 *   ignore it.  Results are identical with and without it; a caller that breaks the
 *   promise (e.g. casts B with fp8_cast_blocks right before the call) may get results
 *   computed from stale weights. */
#define FG_FLAG_STATIC_B 1u

/* The three GEMMs with a caller-owned workspace (device memory, 16-byte aligned, at least
 * fg_workspace_bytes() bytes, zero-filled once before its first use, e.g. with
 * cudaMemsetAsync).  Every kernel leaves the counters at zero again when it finishes, so
 * a workspace can be reused by any number of calls in stream order; calls that may run
 * at the same time (different streams) need different workspaces.  After a call ends
 * with FG_ERR_TIMEOUT (fg_get_device_status) the caller zero-fills its workspace again.
 * workspace == NULL with workspace_bytes == 0 uses the library's own workspace (the _ex
 * entry points); a workspace that is too small is FG_ERR_INVALID_ARG, a misaligned one
 * FG_ERR_ALIGNMENT.  flags: FG_FLAG_* options (0 for none; an unknown bit is
 * FG_ERR_INVALID_ARG).  Everything else is as for the _ex entry points. */
fg_status fp8_gemm_nt_ws(const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                         int M, int N, int K, int fmt_a, int fmt_b, unsigned flags, void* workspace,
                         size_t workspace_bytes, void* stream);
fg_status fp8_gemm_grouped_contiguous_ws(const void* A, const float* sfa, const void* B, const float* sfb,
                                         void* C, const int* m_indices, int M_total, int G, int N, int K,
                                         int fmt_a, int fmt_b, unsigned flags, void* workspace,
                                         size_t workspace_bytes, void* stream);
fg_status fp8_gemm_grouped_masked_ws(const void* A, const float* sfa, const void* B, const float* sfb,
                                     void* C, const int* masked_m, int G, int Mmax, int N, int K,
                                     int fmt_a, int fmt_b, unsigned flags, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* Allocation-free variant of fp8_gemm_nt, for callers that cannot allocate device
 * memory: code running inside another framework's memory pool or a pre-planned
 * static memory budget, code that must not touch the allocator during a
 * latency-critical decode step, or a process that has reserved the whole device
 * up front.  (The pages have no counterpart; it is a deployment convenience.)
 * It takes the same arguments as fp8_gemm_nt, needs no fg_init, and never calls
 * cudaMalloc or cudaFree: its split-K scratch (partial tiles, per-tile counters,
 * a status word; 16 MiB + 64 KiB) is a static device array that every GPU which
 * loads this library holds until the process exits.
 * Limits: M <= 128 (the swap-AB stream-K kernel; larger M returns
 * FG_ERR_UNSUPPORTED) and ceil(N / 128) <= 16384 (else FG_ERR_UNSUPPORTED); the
 * array caps the grid at 16 MiB / (2 * 128 * MP * 4 bytes) CTAs, MP = M rounded
 * up to 32, 64 or 128, so M > 64 runs on at most 128 CTAs.
 * The first call on a device looks up the array's device address (and the
 * tensor-map encoder); make that first call before any stream capture.
 * All calls share the one array: calls that overlap on the GPU (concurrent
 * streams, or other host threads) race and give wrong results.  Each call clears
 * the counters it uses (a memset on `stream`) before its kernel; the partial
 * tiles keep the last call's contents, which no call reads before writing.
 * A wait that times out inside this variant is reported by fg_noalloc_status. */
fg_status fp8_gemm_nt_noalloc(const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                              int M, int N, int K, void* stream);

/* Synchronise `stream`, then read and clear the status word of the
 * allocation-free variant (FG_OK if it was never called on this device). */
fg_status fg_noalloc_status(void* stream);

/* The cast step before the GEMM (the pages leave it to the user: turtlesai.it
 * summary, FP8 casting and the TMA-aligned LHS scale layout are done outside the
 * GEMM kernels).  X holds BF16 values; per block
 *   scale = amax / 448 in fp32 (1 for an all-zero block),
 *   code  = e4m3 round-to-nearest-even of the fp32 quotient x / scale, saturating
 *           at +-448,
 * so that dec(code) * scale approximates x.  Results are exact and deterministic
 * (no accumulation).  X must be finite: a block holding an infinity or a NaN gets
 * unspecified codes and scale.  K % 16 == 0; X and Q 16-byte aligned, scales 4-byte aligned;
 * all pointers are device pointers owned by the caller; nothing is allocated.
 *
 * fp8_cast_rows: the A side (activations).  X is [G][M][K] (G = 1 for a plain
 * [M, K] matrix), Q the e4m3 codes in the same layout, sfa one scale per 1 x 128
 * block of a row in exactly the layout the GEMM entry points read:
 * [G][ceil(K/128)][fg_sfa_ld(M)], column-major per group; its padding rows
 * M .. ld-1 are not written.  G = 0 or M = 0 is a no-op. */
fg_status fp8_cast_rows(const void* X, void* Q, float* sfa, int G, int M, int K, void* stream);

/* fp8_cast_blocks: the B side (weights).  X is [G][N][K], Q the codes, sfb one
 * scale per 128 x 128 block: [G][ceil(N/128)][ceil(K/128)].  G = 0 or N = 0 is a
 * no-op; G and ceil(N/128) must not exceed 65535. */
fg_status fp8_cast_blocks(const void* X, void* Q, float* sfb, int G, int N, int K, void* stream);

/* The two casts with a target format: FG_E4M3 (top = 448, as above) or FG_E5M2
 * (scale = amax / 57344, codes saturating at +-57344); any other value is
 * FG_ERR_INVALID_ARG. */
fg_status fp8_cast_rows_ex(const void* X, void* Q, float* sfa, int G, int M, int K, int fmt, void* stream);
fg_status fp8_cast_blocks_ex(const void* X, void* Q, float* sfb, int G, int N, int K, int fmt, void* stream);

/* Synchronise `stream`, then read and clear the device status word:
 * FG_OK, or FG_ERR_TIMEOUT if some kernel since the last call gave up a wait, or (debug
 * build, libfp8gemm_debug.so, compiled with -DFG_DEBUG) FG_ERR_DEVICE_CHECK if a
 * device-side index check failed.  The first error since the last read wins. */
fg_status fg_get_device_status(void* stream);

/* Human-readable name of a status code (static storage). */
const char* fg_status_string(fg_status status);

/* Kernel selection, process-wide: 0 = automatic (dense M <= 128 takes the
 * swap-AB kernel, scheduled as fg_set_swap_schedule says; everything else follows
 * the tile table -- see fg_tile_plan), 1 = the one-CTA tiled kernel for every
 * dense, contiguous and masked call, 2 = always the swap-AB kernel for dense calls
 * (requires M <= 128), 3 = the CTA-pair kernel (tcgen05 cta_group::2, 256-row
 * tiles over two SMs) for dense and masked calls.  The contiguous layout never
 * takes the CTA pair.  Returns the previous value; an unknown value is ignored. */
int fg_set_dense_path(int path);

/* Output tile width (columns of N per tile) of the tiled and CTA-pair kernels, process-wide:
 * 0 (default) = the tile table, or 128, 192 or 256 to force a width (the CTA-pair kernel has
 * 192 and 256; it takes 192 for a forced 128).  Widths other than these are ignored.
 * Results are identical in every width up to fp32 summation order of split tiles.
 * Returns the previous value. */
int fg_set_tile_n(int bn);

/* Runtime specialisation of the one-CTA tiled kernel (the pages' library compiles its kernels at
 * run time with the GEMM shape as constants: chattools.cn explainer, flashmla.org product page),
 * process-wide, default 0 (off: the ahead-of-time kernels).  With 1, the first call of each
 * shape that takes the one-CTA tiled kernel compiles it with NVRTC for sm_100a with that shape's
 * K blocks, K, N, sfb blocks, tile columns and tile-walk grouping as compile-time constants, from
 * the kernel sources embedded in this library, loads it and caches it (per device and shape);
 * later calls launch it like the ahead-of-time kernel.  Compiling takes about two seconds, so
 * make each shape's first call outside stream capture.  NVRTC (libnvrtc.so.12) and the CUDA
 * headers are looked up at run time under $CUDA_HOME or /usr/local/cuda; without them the call
 * returns FG_ERR_UNSUPPORTED (nothing falls back silently).  Results are bit-identical to the
 * ahead-of-time kernel.  Returns the previous value. */
int fg_set_jit(int enable);

/* Number of runtime-specialised kernels compiled and cached in this process. */
int fg_jit_cache_size(void);

/* Compile (do not load) the runtime-specialised dense tiled kernel for tile width bn (128, 192,
 * 256), num_kb K blocks of 128 and N columns; on success *cubin_bytes is the size of the sm_100a
 * binary.  Needs NVRTC and the CUDA headers but no GPU.  FG_ERR_UNSUPPORTED without them,
 * FG_ERR_CUDA if compilation fails, FG_ERR_INVALID_ARG for bad arguments. */
fg_status fg_jit_compile_check(int bn, int num_kb, int N, size_t* cubin_bytes);

/* Promotion warpgroups of the 256-wide CTA-pair kernel, process-wide: 2 (default) or 4.  With
 * 4 (640 threads per CTA), each SM sub-partition runs four promotion warps, each holding a
 * quarter of its CTA's 128 x 256 accumulators.  Other values are ignored.  Results are
 * identical.  Returns the previous value. */
int fg_set_pair_promotion(int warpgroups);

/* Tile walk of the tiled and CTA-pair kernels, process-wide: 0 (default) = automatic, 1 = groups of
 * m-blocks whose A rows take at most 24 MB, m-block fastest inside a group (B streams through,
 * re-read once per group), 2 = n-block fastest (each m-block's rows are read once while B stays
 * in L2).  Automatic takes 2 when one group's B (N x K bytes) is at most 40 MB, else 1.  Other
 * values are ignored.  Results are identical (each tile is computed the same way).  Returns the
 * previous value. */
int fg_set_tile_order(int order);

/* The kernel and tile width a call of this shape takes on the current device under the
 * current settings, as kernel * 1000 + width: 1xxx the one-CTA tiled kernel, 3xxx the
 * CTA pair, 2000 the small-M swap-AB kernel (dense, M <= 128).  layout: 0 dense, 1
 * contiguous (M = all rows), 2 masked (M = Mmax); G = 1 for dense.  The tile table
 * (automatic settings): N <= 128 -> 128-wide tiles, N <= 192 -> 192, otherwise 256; dense
 * calls take the CTA pair unless its last wave of 256 x 256 tiles would hold at most a
 * quarter of the SM pairs (then the one-CTA kernel, whose stream-K tail splits that wave),
 * contiguous and masked calls the one-CTA kernel.  -1 for invalid arguments or a device
 * without fg_init.  Launches nothing. */
int fg_tile_plan(int layout, int M, int N, int K, int G);

/* Stream-K tail of the tiled kernel (dense M > 128, contiguous, masked), process-wide.
 * The tiles are walked whole in waves over the SMs; when the last wave is partial
 * its tiles are instead split in K over all the CTAs, and a tile split between CTAs
 * is summed (fp32 partials in the library's workspace, in a fixed CTA order, so the
 * result does not depend on timing) by the last CTA to finish it.  The split is taken
 * when the busiest CTA's share of the split units, plus `overhead` K blocks of 128 for
 * publishing partial tiles (default 18) and 2.4 K blocks per piece summed, is at most
 * one whole tile; 0 takes it whenever the last wave is partial, a negative value
 * never.  Returns the previous value.  Results differ from the unsplit walk only in
 * fp32 summation order. */
int fg_set_tiled_streamk(int overhead);

/* Schedule of the small-M (swap-AB) kernel, process-wide.  0 (default): automatic --
 * whole 128-row weight tiles per CTA, stream-K (K blocks split evenly over the CTAs,
 * split tiles summed through global memory by the last CTA to finish), or a cluster
 * split: a thread-block cluster of S CTAs per weight tile, each CTA taking 1/S of the
 * K blocks, the partials summed through distributed shared memory (possible when every
 * tile's cluster can be resident at once and K has at least S blocks of 128); the
 * cheapest by a cost model in K blocks.  -1: never the cluster split.  1: whole tiles,
 * one CTA per tile up to the SM count.  2, 4 or 8: the cluster split with that S
 * wherever it is possible.  Other values are ignored.  All schedules sum in a fixed
 * order.  Returns the previous value. */
int fg_set_swap_schedule(int schedule);

/* K blocks per ring stage of the small-M (swap-AB) and CTA-pair kernels, process-wide.
 * 0 (default) = automatic: 2 when K is a multiple of 128 (the small-M kernel also needs at
 * least four K blocks), each operand copy then moving two K blocks at once -- a CTA's copy
 * rate is bounded by the number of copies in flight more than by their size -- else 1.
 * 1 forces single K blocks; 2 forces pairs wherever K is a multiple of 128.  Any other value
 * is ignored.  Results agree to fp32 summation order (split points of the small-M kernel's
 * K range move to pair boundaries).  Returns the previous value. */
int fg_set_stage_kblocks(int kps);

/* The schedule the small-M kernel takes for a dense call of this shape on the current
 * device under the current setting: S (2, 4 or 8) for the cluster split, 1 for whole
 * tiles per CTA, 0 for stream-K; -1 if M is not in 1..128, N or K is not positive, or
 * fg_init has not been called for the device.  Launches nothing. */
int fg_swap_plan(int M, int N, int K);

/* Failure injection for tests (process-wide, default 0).  With 1, every kernel of
 * fp8_gemm_nt that takes the small-M (swap-AB stream-K) path, and every kernel of
 * fp8_gemm_nt_noalloc, first waits on a barrier that no one arrives at; the bounded
 * wait runs out after about two seconds, the kernel aborts cleanly (its other warps
 * leave their waits, copies in flight are drained, TMEM is freed), writes no output
 * and leaves FG_ERR_TIMEOUT in the device status word for fg_get_device_status()
 * (fg_noalloc_status() for the allocation-free variant).  Nothing faults or traps,
 * and the context stays usable.  Returns the previous value.  Not for production use. */
int fg_debug_set_stall(int enable);

/* Number of GEMM kernel launches the library has issued in this process. */
uint64_t fg_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8GEMM_H */
