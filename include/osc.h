/*
 * libosc: B200 (sm_100a) OSC W4A4 linear layer behind a plain C ABI.
 *
 * The method is the one of the OSC page, "W4A4量化技术：OSC框架如何实现高效LLM部署"
 * (coreui.cn/article/2607942.html): a static, offline suppression table names one outlier
 * channel per G-wide channel group (§3.1, Algorithm 1); at run time that value is moved into
 * a high-precision buffer B and zeroed, the zeroed tensor is microscaled to 4 bits (§3.2,
 * Figure 2), and the layer output is the dual-path product
 *     Y = (Q_X (x) Q_W) * S + B * W_L                         (§3.2)
 * with W_L the bf16 weight rows of the table's channels (§3.3). Low-clustering inputs (W2)
 * fall back to an FP8 microscaled product (§2.3, §4); MoE expert layers use a grouped form
 * (§1, §5.2). Element formats are OCP MX: E2M1 (or E4M3) elements with one E8M0
 * power-of-two scale per block.
 *
 * Conventions for every entry point:
 *   - Tensors are caller-allocated DEVICE memory (e.g. from PyTorch); the library never
 *     allocates or frees memory and never synchronizes the stream, except osc_status.
 *   - Every call is asynchronous on the given stream (a cudaStream_t; NULL = legacy stream).
 *   - bf16 values are passed as uint16_t bit patterns; 4-bit and 8-bit codes as uint8_t.
 *   - All pointers must be 16-byte aligned (cudaMalloc / PyTorch allocations are).
 *   - Inputs must be finite (no NaN / Inf).
 *   - Return value: OSC_OK (0) or a negative OSC_ERR_* code; nothing is launched on error.
 *     A call with zero rows (M = 0) does nothing and returns OSC_OK; its pointers may be NULL.
 *     Errors found by a kernel while it runs (a table entry >= G, more entries than K_L,
 *     a bounded wait that ran out) are recorded in a per-device status word that
 *     osc_status() reads and clears. The word is shared by every stream and host thread
 *     using the device in this process; it keeps the first error recorded since it was last
 *     cleared. After OSC_ERR_TIMEOUT, every output written since the last clean osc_status
 *     is undefined (the kernel that ran out stopped part way and returned).
 *   - osc_set_tile_n and osc_set_cta_pair change process-wide launch choices; they are
 *     tuning and test knobs, not meant to be flipped while other threads issue calls.
 *
 * Shapes: X is M x K bf16 row-major (tokens x input channels); W is N x K bf16 row-major
 * (output x input channels, the layout of a PyTorch Linear weight); Y is M x N bf16.
 * K must be a multiple of 256. N must be a multiple of 16. G is 16, 32 or 64.
 *
 * Layouts the calls exchange (all row-major):
 *   QX / QW  (MXFP4) rows x K/2 bytes: element k of a row in byte k/2, even k in the low nibble.
 *            (MXFP8) rows x K bytes, one E4M3 code per element.
 *            Codes keep the sign of the input even when the magnitude rounds to zero.
 *   SX / SW  E8M0 scale bytes (e + 127) in the tensor-core scale layout: 512-byte atoms of
 *            128 rows x 4 slots; slot s of row r lives at byte
 *              ((r/128) * (K/V/4) + s/4) * 512 + (r%32)*16 + ((r%128)/32)*4 + s%4
 *            with V = 16 for G = 16 and V = 32 otherwise (G = 64 stores its one exponent in
 *            both 32-slots of the group). Rows are padded to a multiple of 128; the pad
 *            rows hold 0. Size: osc_scale_bytes().
 *            Shared exponent e = floor(log2(amax)) - 2 (E2M1) or - 8 (E4M3), clamped to
 *            [-127, 127]; an all-zero block gets e = -127.
 *   L        int8, K/G x R entries (R = 1..3 protected channels per group): slot r of group k
 *            at L[k*R + r], the local channel 0..G-1 of an outlier, or -1.
 *   B        M x K_L bf16: column i holds the i-th table entry >= 0 in (group, slot) order;
 *            columns past the entry count are 0. Entries are moved out in that order, so a
 *            channel named twice in a group gives its value once and 0 the second time.
 *   W_L      N x K_L bf16: W_L[n][i] = W[n][channel of table entry i]; pad columns 0.
 *   K_L      the compensation width: the number of table entries rounded up to a multiple
 *            of 16 (osc_table_kl), or any larger multiple of 16.
 */
#ifndef OSC_H_
#define OSC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define OSC_API __attribute__((visibility("default")))
#else
#define OSC_API
#endif

typedef struct CUstream_st* osc_stream_t; /* same type as cudaStream_t */

enum {
  OSC_OK = 0,
  OSC_ERR_ARG = -1,      /* null pointer, negative or unsupported size */
  OSC_ERR_ALIGN = -2,    /* pointer not 16-byte aligned, K % 256 != 0, N % 16 != 0, K_L % 16 != 0 */
  OSC_ERR_G = -3,        /* G not in {16, 32, 64} */
  OSC_ERR_CUDA = -4,     /* a CUDA runtime/driver call failed; see osc_last_cuda_error() */
  OSC_ERR_TIMEOUT = -5,  /* (from osc_status) a kernel's bounded wait ran out */
  OSC_ERR_TABLE = -6,    /* (from osc_status) a table entry >= G or more entries than K_L */
  OSC_ERR_DEVICE = -7,   /* the current device is not an sm_100 GPU */
  OSC_ERR_SCRATCH = -8   /* (osc_linear_splitk_noalloc) the call needs more than its fixed scratch */
};

/* Library version string. */
OSC_API const char* osc_version(void);
/* Human-readable text for an OSC_* code. */
OSC_API const char* osc_error_string(int code);
/* The cudaError_t value behind the last OSC_ERR_CUDA returned on this thread. */
OSC_API int osc_last_cuda_error(void);

/* Bytes of a scale buffer for `rows` rows of K channels with group size G (G = 16, 32, 64),
 * or for the MXFP8 path when G == 0. Returns 0 on invalid arguments. */
OSC_API size_t osc_scale_bytes(int rows, int K, int G);

/* K_L for a table held in HOST memory: count of its n entries (K/G x R) that are >= 0, rounded
 * up to 16. */
OSC_API int osc_table_kl(const int8_t* L_host, int n);

/* §3.1 Algorithm 1 (offline), one (position, layer): S x K calibration activations Xcal
 * -> L (K/G entries, device). alpha is the page's threshold (default 5); min_hits is the
 * fewest events a channel needs to be protected (default 5). An event of group k on token t
 * is the channel j_t of largest |x| (lowest j on ties) when G*|x_max| >= alpha * sum|x_j|
 * (sum in fp32 over ascending j, comparison in fp64); L[k] is the channel with the most
 * events (lowest on ties) if it has >= min_hits, else -1. */
OSC_API int osc_build_table(const uint16_t* Xcal, int S, int K, int G, float alpha, int min_hits,
                    int8_t* L, osc_stream_t stream);

/* §6 multi-outlier protection (up to R = 1..3 channels per group, "for extreme cases"; the
 * page gives no procedure): R rounds of the osc_build_table rule, round r counting events with
 * the channels of rounds 0 .. r-1 read as zero (what extraction leaves of the group), so a
 * further channel is protected only while it stays a consistent outlier once the stronger ones
 * are out. L receives K/G x R entries (device), slot r of group k at L[k*R + r]; once a round
 * finds no channel for a group its later slots are -1. R = 1 is osc_build_table. */
OSC_API int osc_build_table_multi(const uint16_t* Xcal, int S, int K, int G, float alpha, int min_hits,
                                  int R, int8_t* L, osc_stream_t stream);

/* §2.2 clustering density of a table on S x K activations X (device), with the event of
 * osc_build_table: n_total[k] counts group k's outlier events over the S tokens and n_hit[k]
 * those whose channel is L[k] (0 when L[k] = -1), so C_k = n_hit[k] / n_total[k]. L, n_hit
 * and n_total are device arrays of K/G entries (int8, int32, int32). A table entry >= G is
 * recorded in the status word (OSC_ERR_TABLE from osc_status) and counts no hits. */
OSC_API int osc_density(const uint16_t* X, int S, int K, int G, float alpha, const int8_t* L,
                        int* n_hit, int* n_total, osc_stream_t stream);

/* Tiers of §2.3, chosen from the density of a module input. */
enum {
  OSC_TIER_FP8 = 0,   /* C < 35 %: MXFP8 fallback (§4) */
  OSC_TIER_MID = 1,   /* 35 % <= C <= 60 %: static protection still helps (OSC W4A4) */
  OSC_TIER_HIGH = 2   /* C > 60 %: static channel protection (OSC W4A4) */
};

/* HOST logic on the counts of osc_density (host arrays, Kg entries): C = mean over the groups
 * with events (n_total > 0) of n_hit / n_total, summed in double over ascending k; *c_bar
 * (may be NULL) receives it. Returns the tier above, or OSC_ERR_ARG for a negative count or
 * n_hit > n_total (the arrays may be NULL when Kg = 0). With no events at all, *c_bar is NaN and the result is OSC_TIER_HIGH
 * (nothing escapes the table; with an empty table OSC is plain MXFP4). */
OSC_API int osc_select_tier(const int* n_hit, const int* n_total, int Kg, double* c_bar);

/* §6 "dynamic group size" (HOST logic): the group size of one module from its clustering
 * density measured with tables built at G = 16, 32 and 64, c_bar[0..2] in that order (NaN
 * where a G saw no events, as osc_select_tier reports it). The page names the idea without a
 * rule; this one keeps the page's tiers at its default G = 32 and moves G only where static
 * protection holds at the high tier: the largest G whose C is above 60 % (fewer scales and
 * table entries, the fastest product in Table 2); if no G is that high, G = 32 with its own
 * tier. Returns 16, 32 or 64, or 0 when the module takes the MXFP8 fallback (G = 32 in the
 * fallback tier); *tier (may be NULL) receives the tier of the choice. OSC_ERR_ARG if
 * c_bar is NULL. */
OSC_API int osc_select_group_size(const double* c_bar, int* tier);

/* §3.2, Figure 2 (online): extraction + zeroing through the table, then MXFP4 quantization
 * of the zeroed tensor. X (M x K bf16) -> QX (M x K/2), SX (osc_scale_bytes(M, K, G)),
 * B (M x K_L bf16). L: K/G x R entries (R = 1..3 protected channels per group, see L below),
 * or NULL (no table: plain MXFP4; then K_L must be 0, B may be NULL and R is not used, pass 1).
 * X is not modified. With a table, K/G x R may be at most 4096. */
OSC_API int osc_quantize(const uint16_t* X, int M, int K, int G, const int8_t* L, int R, int K_L,
                 uint8_t* QX, uint8_t* SX, uint16_t* B, osc_stream_t stream);

/* Figure 2 (§3.2) with the step that produces the projection's input: RMSNorm of each row,
 * then the osc_quantize of the normalized row, in one pass over X (the normalized rows are
 * never written out). X: M x K bf16 activations, gamma: K bf16 weights, eps >= 0. Per row, in
 * fp32 with every operation rounded to nearest even: the squares of each 32-channel block
 * summed in ascending order; the block sums padded with zeros to a power of two and combined
 * pairwise (s_b += s_{b+h}, h = P/2 .. 1); inv = 1 / sqrt(sum / K + eps); the normalized value
 * bf16((x * inv) * gamma). Outputs and table arguments as osc_quantize (the table comes from
 * calibration rows that were normalized the same way). K must be at most 6144. */
OSC_API int osc_rmsnorm_quantize(const uint16_t* X, const uint16_t* gamma, float eps, int M, int K, int G,
                                 const int8_t* L, int R, int K_L, uint8_t* QX, uint8_t* SX, uint16_t* B,
                                 osc_stream_t stream);

/* §3.3 weight side (offline): W (N x K bf16) -> QW (N x K/2), SW (osc_scale_bytes(N, K, G))
 * quantized with no table (its outlier columns meet zeroed activations), and
 * W_L (N x K_L bf16) gathered through L (K/G x R entries, device; may be NULL when K_L == 0). */
OSC_API int osc_prepare_weight(const uint16_t* W, int N, int K, int G, const int8_t* L, int R, int K_L,
                       uint8_t* QW, uint8_t* SW, uint16_t* WL, osc_stream_t stream);

/* §3.2 equation for Y: Y (M x N bf16, round to nearest even from the fp32 accumulator)
 *   = sum_b 2^(eX+eW) sum_{i in b} qX qW  +  B * W_L^T.
 * Yf32 (M x N fp32) may be NULL; when given it receives the fp32 accumulator as well
 * (a checking aid; it slows the call down). B and WL may be NULL when K_L == 0. */
OSC_API int osc_linear(const uint8_t* QX, const uint8_t* SX, const uint16_t* B,
               const uint8_t* QW, const uint8_t* SW, const uint16_t* WL,
               int M, int N, int K, int G, int K_L, uint16_t* Y, float* Yf32,
               osc_stream_t stream);

/* Figure 2 and the §3.2 equation in one call: osc_quantize(X, M, K, G, L, R, K_L, QX, SX, B)
 * then the product on the same stream: osc_linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y,
 * Yf32) when workspace is NULL, else osc_linear_splitk(..., Y, Yf32, workspace,
 * workspace_bytes) (see below: the split applies at M <= 16). Same arguments, outputs and errors
 * as the two calls (every argument is checked before either kernel is launched; QX, SX and B
 * are written as by osc_quantize), and results identical to them. Because the library issues
 * both kernels back to back, the general product may start reading QW, SW and WL (which the
 * quantize does not write) before the quantize has finished. As for any call, the weight
 * operands must be complete before the call is issued. */
OSC_API int osc_quantize_linear(const uint16_t* X, int M, int K, int G, const int8_t* L, int R, int K_L,
                                uint8_t* QX, uint8_t* SX, uint16_t* B, const uint8_t* QW, const uint8_t* SW,
                                const uint16_t* WL, int N, uint16_t* Y, float* Yf32, float* workspace,
                                size_t workspace_bytes, osc_stream_t stream);

/* The same with the RMSNorm-fused quantize: osc_rmsnorm_quantize(X, gamma, eps, ...) then
 * osc_linear on the same stream, in one call, with the arguments, outputs and errors of the two
 * calls (K at most 6144); the product may start reading QW, SW and WL before the quantize ends. */
OSC_API int osc_rmsnorm_quantize_linear(const uint16_t* X, const uint16_t* gamma, float eps, int M, int K, int G,
                                        const int8_t* L, int R, int K_L, uint8_t* QX, uint8_t* SX, uint16_t* B,
                                        const uint8_t* QW, const uint8_t* SW, const uint16_t* WL, int N,
                                        uint16_t* Y, float* Yf32, osc_stream_t stream);

/* The product of osc_linear for few token rows, with the weight stream split over more SMs.
 * For M <= 16 (decoding) the product is weight-bound: every call reads all of QW, SW and W_L,
 * and osc_linear gives each 128-row weight tile one SM. osc_linear_splitk computes the product
 * transposed (the weight tile as the 128-row tensor-core operand, the token rows as its
 * 16-wide side) and splits each tile's K range over S SMs: each part writes its fp32 partial
 * product (M x N) into `workspace`, and a second kernel on the same stream adds the S partials
 * in a fixed order (part 0 first) and rounds to bf16, so Y does not depend on timing.
 * Arguments as osc_linear, plus workspace: caller-allocated device memory of workspace_bytes
 * bytes (16-byte aligned). Its contents need no initial value and are left undefined; calls
 * that share a workspace must not overlap on the GPU. osc_linear_workspace_bytes(M, N, K, K_L)
 * gives the bytes the split needs, 0 when no split applies (M > 16, or the weight tiles
 * alone fill the SMs); when no split applies or workspace_bytes is smaller, the call runs
 * exactly as osc_linear. */
OSC_API size_t osc_linear_workspace_bytes(int M, int N, int K, int K_L);
OSC_API int osc_linear_splitk(const uint8_t* QX, const uint8_t* SX, const uint16_t* B,
                              const uint8_t* QW, const uint8_t* SW, const uint16_t* WL,
                              int M, int N, int K, int G, int K_L, uint16_t* Y, float* Yf32,
                              float* workspace, size_t workspace_bytes, osc_stream_t stream);

/* Allocation-free form of osc_linear_splitk (the OSC page has no counterpart: this is a
 * deployment convenience of this library). Some callers cannot allocate device memory at all:
 * plugins of an inference engine that owns every device buffer and hands a plugin only its
 * inputs and outputs, or serving loops that forbid allocation after start-up (an allocation
 * there could fail under fragmentation or stall other streams). They cannot provide the
 * workspace osc_linear_splitk needs, so this entry point keeps the fp32 partials in one fixed
 * buffer inside the library instead: OSC_NOALLOC_SCRATCH_BYTES (16 MiB) of device memory that
 * every GPU which loads the library holds until the process exits. Arguments and results as
 * osc_linear_splitk without the workspace; the library still allocates nothing, and the caller
 * passes inputs and outputs as usual.
 *   - The first call on a device looks up the buffer's device address (once per device, with
 *     that device current); make that first call before any stream capture.
 *   - A call whose split needs more partial bytes than the buffer holds (S x M x N x 4, see
 *     osc_linear_workspace_bytes) returns OSC_ERR_SCRATCH and launches nothing; calls that
 *     need no split (M > 16, or one part per weight tile) use no scratch.
 *   - Every call shares the one buffer and it keeps the last call's contents; nothing in it
 *     needs to start at zero (each call writes every partial it reads). Calls that overlap on
 *     the GPU (different streams, or different host threads without ordering) race on it. */
#define OSC_NOALLOC_SCRATCH_BYTES (16u << 20)
OSC_API int osc_linear_splitk_noalloc(const uint8_t* QX, const uint8_t* SX, const uint16_t* B,
                                      const uint8_t* QW, const uint8_t* SW, const uint16_t* WL,
                                      int M, int N, int K, int G, int K_L, uint16_t* Y, float* Yf32,
                                      osc_stream_t stream);

/* §4 FP8 fallback, quantize side: X (M x K bf16) -> QX8 (M x K E4M3 codes),
 * SX (osc_scale_bytes(M, K, 0)); per-32 E8M0 scales, no separation. Also used for the
 * weights of the fallback. */
OSC_API int osc_quantize_fp8(const uint16_t* X, int M, int K, uint8_t* QX8, uint8_t* SX,
                     osc_stream_t stream);

/* §4 FP8 fallback product: Y = sum_b 2^(eX+eW) sum_{i in b} qX qW over E4M3 codes. */
OSC_API int osc_linear_fp8_fallback(const uint8_t* QX8, const uint8_t* SX, const uint8_t* QW8,
                            const uint8_t* SW, int M, int N, int K, uint16_t* Y, float* Yf32,
                            osc_stream_t stream);

/* ---- grouped (MoE) form, §1 and §5.2 (Qwen3-30B-A3B expert layers) -------------------
 * Tokens arrive sorted by expert: expert e owns rows off[e] .. off[e+1] of X. The grouped
 * calls work on a PADDED row space in which expert e's rows start at poff[e], a multiple of
 * 128, so that every 128-row block belongs to one expert (mblock_expert[b] = e).
 * osc_grouped_plan fills the three host arrays from per-expert counts. */

/* counts (E entries, host) -> off (E+1), poff (E+1), mblock_expert (poff[E]/128 entries),
 * all host arrays; returns the padded row count poff[E], or a negative code. mblock_expert
 * may be NULL to query the size first. */
OSC_API int osc_grouped_plan(const int* counts, int E, int* off, int* poff, int* mblock_expert,
                     int mblock_capacity);

/* Per-expert extraction + MXFP4 quantization. X: T x K bf16 (device), T = off[E] the routed
 * rows (the value of off[E] on the host, passed so that the call needs no copy back). off, poff,
 * mblock_expert: device copies of the plan. L: E x K/G x R (device), expert e's table at
 * e*K/G*R.
 * Outputs over the padded rows: QX (Mp x K/2), SX (osc_scale_bytes(Mp, K, G)),
 * B (Mp x K_L bf16, K_L a common width >= every expert's entry count); pad rows are 0.
 * E x K/G x R may be at most about 68000 table entries (they are staged in shared memory). */
OSC_API int osc_quantize_grouped(const uint16_t* X, int T, int E, const int* off, const int* poff,
                         const int* mblock_expert, int Mp, int K, int G, const int8_t* L, int R,
                         int K_L, uint8_t* QX, uint8_t* SX, uint16_t* B, osc_stream_t stream);

/* Per-expert dual-path product over the padded rows. QW: E x N x K/2, SW: E blocks of
 * osc_scale_bytes(N, K, G), WL: E x N x K_L (each expert's W_L padded to the common K_L),
 * kl: E compensation widths (device, multiples of 16, <= K_L; NULL = K_L for all).
 * Y: Mp x N bf16 (pad rows receive 0). */
OSC_API int osc_linear_grouped(const uint8_t* QX, const uint8_t* SX, const uint16_t* B,
                       const uint8_t* QW, const uint8_t* SW, const uint16_t* WL,
                       const int* mblock_expert, const int* kl, int E, int Mp, int N, int K,
                       int G, int K_L, uint16_t* Y, float* Yf32, osc_stream_t stream);

/* Reads and clears the current device's status word in one atomic exchange on `stream`, then
 * synchronizes `stream`. Returns OSC_OK, OSC_ERR_TIMEOUT or OSC_ERR_TABLE; *raw (may be NULL)
 * gets the raw device code. An error that a kernel on another stream records while this call
 * runs is either returned by it or kept for the next call. */
OSC_API int osc_status(int* raw, osc_stream_t stream);

/* Failure-detection self-test (not part of the OSC method): launches one kernel whose bounded
 * wait on a barrier that nothing signals runs out after limit_us microseconds (1 .. 1000000).
 * The timeout is recorded in the status word exactly as a stalled kernel pipeline records it,
 * so the next osc_status returns OSC_ERR_TIMEOUT. No fault, trap or unbounded wait. */
OSC_API int osc_selftest_timeout(int limit_us, osc_stream_t stream);

/* Tile width of the tensor-core kernels: 0 = automatic (default), 128 or 256. Applies to
 * calls made afterwards from any thread. Returns the previous value, or OSC_ERR_ARG. */
OSC_API int osc_set_tile_n(int bn);

/* CTA grouping of the tensor-core kernels: -1 = automatic (default), 1 = one CTA per
 * 128-row tile, 2 = a 2-CTA cluster per 256-row tile (tile width 256; dense calls only).
 * Returns the previous value, or OSC_ERR_ARG. */
OSC_API int osc_set_cta_pair(int mode);

#ifdef __cplusplus
}
#endif

#endif /* OSC_H_ */
