/*
 * bonsai.h -- C ABI of libbonsai, the B200 (sm_100a) ternary linear layer of
 * Bonsai 2-style ternary language models.
 *
 * The layer computes  y = x' . Wdeq^T  where
 *   - W is N x K (out x in) with trits t in {-1, 0, +1} and one FP16 scale per
 *     run of 128 weights along K:  Wdeq[n][k] = s[n][k/128] * t[n][k];
 *     source: "27B 模型压到 5.95GB，推理能力还保住 98%" (allhereai.com), the
 *     paragraph describing the method (ternary weights, a shared FP16 scale per
 *     128 weights, a block Hadamard rotation folded into storage);
 *   - x' = blockdiag(Hn) x is the online block-Hadamard rotation of the
 *     activations, Hn = H_128 / sqrt(128) with H_128 the Sylvester matrix
 *     (Hn[i][j] = (-1)^popcount(i & j) / sqrt(128)), applied to each run of 128
 *     activations starting at a multiple of 128; sources: the same page, the
 *     paragraph on running the files (a Hadamard activation runtime is needed,
 *     without it the output is garbage), and "Bonsai 2，把27B压进6个G"
 *     (10100.com), section 它怎么做到的 (the input must get the matching transform).
 *
 * Layouts (all row-major, all buffers owned by the caller):
 *   x       M x K   FP16 (IEEE binary16 bit patterns in uint16_t)
 *   y       M x N   FP16, round-to-nearest-even from an FP32 accumulator
 *   scales  N x K/128  FP16 (N x K/64 for BONSAI_FMT_PQ2_0_G64)
 *   trits   N x K   int8 in {-1, 0, +1}
 *   packed  the plane of one of the formats below: the two packings of the
 *           allhereai.com page (paragraph on the two file packings) and two
 *           variants the wmrh.cn page names:
 *     BONSAI_FMT_PTQ1_0  "compact trits", 1.75 bits/weight with the scale:
 *         row n, group g (128 weights) occupies 26 bytes at (n*K/128 + g)*26;
 *         byte b < 25 holds weights 128g+5b .. 128g+5b+4, byte 25 the last
 *         three, as  byte = sum_i (t_i + 1) * 3^i  (first weight least
 *         significant; padding digits zero, so byte 25 < 27; bytes >= 243
 *         are invalid).  Trit plane size N * K/128 * 26 bytes.
 *     BONSAI_FMT_PQ2_0   one trit per 2-bit slot, 2.125 bits/weight with the
 *         scale: weight k of row n is code t+1 in bits 2(k%4), 2(k%4)+1 of byte
 *         n*K/4 + k/4 (code 3 is invalid).  Trit plane size N * K/4 bytes.
 *     BONSAI_FMT_Q1_0    the 1-bit sibling of the wmrh.cn page (section 核心观点,
 *         ~1.125 bits/weight; section 关键机制, weights in {-1, +1} with an FP16
 *         group scale): weight k of row n is bit k%8 of byte n*K/8 + k/8, 1 for +1
 *         and 0 for -1 (every byte is valid).  Plane size N * K/8 bytes.  Same
 *         scale plane and the same rotation of x as the ternary packings.
 *     BONSAI_FMT_PQ2_0_G64  the PQ2_0 plane (same bytes, packed by bonsai_pack_pq2)
 *         with one FP16 scale per 64 weights: scales is N x K/64, scale g covering
 *         weights 64g .. 64g+63 of its row (the pages' Q2_0_g64; wmrh.cn page, 快速上手
 *         and 后端支持现状).  2.25 bits/weight with the scales.
 *
 * Conventions for every entry point:
 *   - Pointers are CUDA device pointers (any allocator) and must be 16-byte
 *     aligned; sizes are element counts.  K must be a positive multiple of 128;
 *     M and N must be >= 1 (M = 0 or N = 0 is accepted and launches nothing).
 *   - stream is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Calls are asynchronous on it.  The return value reports argument
 *     validation and launch only: on a non-zero return nothing was launched
 *     (validation) or the launch failed (BONSAI_ERR_CUDA).  Faults inside a
 *     kernel surface at the caller's next synchronisation.
 *   - The library keeps one internal workspace per device (FP32 split-K
 *     partials and an FP16 copy of x' for the prefill GEMM).  It is allocated
 *     with cudaMalloc on the first call that needs it, grown when a larger
 *     call arrives (after a device synchronisation), and released by
 *     bonsai_shutdown().  Calls that use it must not overlap on the GPU (keep
 *     them on one stream); bonsai_reserve() sizes it ahead of stream capture.
 *   - Invalid codes in a packed plane (PTQ1_0 bytes >= 243, PQ2_0 code 3)
 *     produce unspecified output values but never out-of-bounds accesses.
 *   - Every wait inside a kernel (a barrier on a copy in flight, a hand-over
 *     between CTAs of the same grid) gives up after a bounded number of polls;
 *     the call then writes NaN to the outputs it could not finish instead of
 *     hanging the GPU, and sets a bit in the device status word that
 *     bonsai_device_status() reads.  Hand-over data carries the number of the call
 *     that wrote it, so a piece that arrives after its reader gave up is never taken
 *     for a later call's: the next call runs normally.
 */
#ifndef BONSAI_H
#define BONSAI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BONSAI_FMT_PTQ1_0 = 1,
    BONSAI_FMT_PQ2_0 = 2,
    BONSAI_FMT_Q1_0 = 3,
    BONSAI_FMT_PQ2_0_G64 = 4
} bonsai_fmt;

typedef enum {
    BONSAI_OK = 0,
    BONSAI_ERR_NULL = -1,   /* a required pointer is NULL                          */
    BONSAI_ERR_SHAPE = -2,  /* M, N or K negative, K not a multiple of 128, or too large */
    BONSAI_ERR_FMT = -3,    /* unknown packing format                             */
    BONSAI_ERR_ALIGN = -4,  /* a pointer is not 16-byte aligned                   */
    BONSAI_ERR_CUDA = -5,   /* a CUDA runtime call or kernel launch failed        */
    BONSAI_ERR_ARCH = -6,   /* the current device is not compute capability 10.0  */
    BONSAI_ERR_NOMEM = -7,  /* the internal workspace could not be allocated      */
    BONSAI_ERR_ALGO = -8,   /* the requested kernel cannot run this shape         */
    BONSAI_ERR_TOO_LARGE = -9 /* beyond the fixed scratch of bonsai_ternary_linear_noalloc */
} bonsai_status;

/* Kernel selection for bonsai_ternary_linear_algo (bonsai_ternary_linear uses AUTO). */
typedef enum {
    BONSAI_ALGO_AUTO = 0,
    BONSAI_ALGO_SIMPLE = 1,  /* one warp per output row; any M (slow, plain)              */
    BONSAI_ALGO_GEMV = 2,    /* batch-1 lookup-table GEMV with split-K; M == 1 only       */
    BONSAI_ALGO_SKINNY = 3,  /* register-dequant tensor-core kernel; 1 <= M <= 16         */
    BONSAI_ALGO_GEMM = 4,    /* tcgen05/TMEM prefill GEMM on FP16 tiles; any M            */
    BONSAI_ALGO_IMMA = 5     /* GEMV on the integer tensor cores, PQ2_0 and PQ2_0 g64:
                                M == 1 (K <= 24576), M == 2 (K <= 12288), and for
                                PQ2_0 M == 3 (K <= 6144)                                  */
} bonsai_algo;

/* Library version, (major << 16) | (minor << 8) | patch. */
int bonsai_version(void);

/* Human-readable text for a bonsai_status value (static storage). */
const char *bonsai_status_string(int status);

/* BONSAI_OK if the current CUDA device is an sm_100 part the library was compiled for,
 * BONSAI_ERR_ARCH if it is another architecture, BONSAI_ERR_CUDA if there is no
 * usable device. */
int bonsai_check_device(void);

/* Bytes of the packed trit plane for N x K weights (scales excluded: they are
 * N * K/128 FP16 values, N * K/64 for BONSAI_FMT_PQ2_0_G64).  Returns BONSAI_ERR_SHAPE / BONSAI_ERR_FMT
 * (negative) on a bad argument. */
int64_t bonsai_packed_bytes(int fmt, int64_t N, int64_t K);

/* Packs N x K trits into the PTQ1_0 plane (layout above).  A trit outside
 * {-1, 0, +1} makes its byte 0xFF, an invalid code, so a bad input is
 * detectable by bonsai_unpack.  Packing is an offline step; its cost is not on
 * the inference path.  Source: allhereai.com page, paragraph on the packings. */
int bonsai_pack_ptq1(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K, void *stream);

/* Packs N x K trits into the PQ2_0 plane (layout above).  A trit outside
 * {-1, 0, +1} is stored as the invalid code 3.  Same source. */
int bonsai_pack_pq2(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K, void *stream);

/* Packs N x K weights into the Q1_0 plane (layout above): +1 -> bit 1, any other
 * value -> bit 0 (-1).  Source: wmrh.cn page, sections 核心观点 and 关键机制. */
int bonsai_pack_q1(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K, void *stream);

/* Unpacks a plane of format fmt back into N x K int8 trits.  Invalid codes
 * unpack to -128 (every trit of an invalid PTQ1_0 byte).  Test hook: it makes
 * the packed layout checkable byte for byte. */
int bonsai_unpack(int fmt, const uint8_t *packed, int8_t *trits, int64_t N, int64_t K,
                  void *stream);

/* x_out = blockdiag(Hn) x for an M x K FP16 matrix (the rotation defined above),
 * computed in FP32 and rounded to FP16 (nearest even).  x_out may equal x (in
 * place) but must not otherwise overlap it.  This is the same transform
 * bonsai_ternary_linear applies internally; it is exported for callers that
 * keep rotated activations and as a test hook. */
int bonsai_hadamard128(const uint16_t *x, uint16_t *x_out, int64_t M, int64_t K, void *stream);

/* y = x' . Wdeq^T (definitions above) for un-rotated FP16 x: the Hadamard
 * rotation of x is applied inside the call.  Dispatch on M: M == 1 -> the
 * integer tensor-core GEMV (PQ2_0 and PQ2_0 g64, K <= 24576, and a grid of at most one
 * CTA per SM: up to about 14,000 items of 32 rows x 512 weights on 148 SMs) or the lookup-table GEMV
 * (PTQ1_0, Q1_0), 2 <= M <= 16 -> skinny tensor-core kernel (PQ2_0, PQ2_0 g64,
 * Q1_0), otherwise (and for PTQ1_0 at 2 <= M <= 16) the tcgen05 GEMM.  The
 * integer GEMV holds each 128-group of x' as 16-bit fixed point with a power-of-two
 * scale (|x~| <= 2^14) before the exact integer products; the other kernels round
 * x' to FP16 (GEMM, skinny) or keep it in FP32 (lookup tables, plain kernel).  y must
 * not overlap x, packed or scales.  Source of the operation: allhereai.com page,
 * method paragraph and packings paragraph. */
int bonsai_ternary_linear(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                          uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, void *stream);

/* As bonsai_ternary_linear with an explicit kernel choice (bonsai_algo) and an
 * explicit split-K factor for the skinny kernel (0 = automatic, 1 = no split,
 * otherwise the number of K chunks, clamped to what the shape allows).  For
 * BONSAI_ALGO_GEMM the same argument picks the M tile instead: 1 = 128 rows per CTA,
 * 2 = 256 rows (two TMEM accumulators sharing each expanded weight tile), 3 = CTA
 * pairs (clusters of two SMs issuing 256-row tcgen05 MMAs together, each SM expanding
 * half of every weight tile; an explicit choice only), 0 = automatic (1 or 2).  For
 * BONSAI_ALGO_GEMV it picks the schedule: 1 = each CTA walks all K slices of its rows
 * (no split-K), >= 2 = one 512-wide K slice per CTA with split-K partials, 0 =
 * automatic.  BONSAI_ALGO_IMMA ignores it (its work split is fixed
 * by the shape and the SM count, so results are bitwise repeatable).
 * Returns BONSAI_ERR_ALGO if the chosen kernel cannot run the shape (e.g.
 * BONSAI_ALGO_GEMV with M > 1, or BONSAI_ALGO_IMMA on a shape whose grid would not fit
 * on the current device at once, the limit the automatic choice also applies).  For
 * measurement and testing of each kernel. */
int bonsai_ternary_linear_algo(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                               uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, int algo,
                               int split_k, void *stream);

/* The SwiGLU step of the MLP after a fused gate/up projection: for y, the M x 2F FP16
 * output of a linear layer whose weight rows 0 .. F-1 are the gate projection and
 * F .. 2F-1 the up projection, h[m][f] = silu(y[m][f]) * y[m][F + f] with
 * silu(z) = z / (1 + e^-z), computed in FP32 and rounded to FP16 (nearest even).  h is
 * M x F; y and h must not overlap.  Source of the fused gate/up projection: the
 * 27B-class layer shapes (d = 5120, ffn = 17408, gate/up N = 34816). */
int bonsai_swiglu(const uint16_t *y, uint16_t *h, int64_t M, int64_t F, void *stream);

/* The fused gate/up linear layer followed by SwiGLU: packed and scales hold 2F weight rows
 * (gate rows first, then up rows: the N = 2F plane of bonsai_ternary_linear) and h gets
 * the M x F result of bonsai_swiglu applied to their product with x'.  On the integer
 * tensor-core GEMV (PQ2_0 and PQ2_0 g64 at the batches and K it takes: see
 * BONSAI_ALGO_IMMA) and the prefill GEMM the step runs in the kernel's epilogue on the
 * FP32 sums; the lookup-table GEMV, the skinny and the plain kernel write the product to
 * the library's workspace in FP16 and bonsai_swiglu follows. */
int bonsai_ternary_linear_swiglu(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                                 uint16_t *h, int64_t M, int64_t F, int64_t K, int fmt, void *stream);

/* Number of kernels one bonsai_ternary_linear_algo call with these arguments launches
 * on the current device (the lookup-table GEMV: 1, or 2 when its split-K partials are
 * summed by a second kernel; the integer tensor-core GEMV: 1; the other kernels: 2,
 * the rotation pass and the kernel),
 * or a negative bonsai_status.  Launches nothing. */
int bonsai_launch_count(int64_t M, int64_t N, int64_t K, int fmt, int algo, int split_k);

/* Grows the calling device's workspace so that calls up to M x N x K (any
 * format and kernel) need no further allocation; call before capturing calls
 * into a CUDA graph.  Synchronises the device if it reallocates. */
int bonsai_reserve(int64_t M, int64_t N, int64_t K);

/* Batch-1 ternary linear layer that allocates nothing.
 *
 * Some callers cannot call cudaMalloc: code that runs while a CUDA graph is being
 * captured, allocators that must own every byte on the device, or hosts that forbid
 * allocation after start-up.  This entry point computes the same y as
 * bonsai_ternary_linear for M == 1 with the split-K lookup-table GEMV, but takes that
 * kernel's scratch -- one FP32 partial sum per (512-weight K slice, output row) -- from
 * one fixed array in device memory that is part of the library image, instead of the
 * per-device workspace.  It never calls cudaMalloc, cudaFree or any allocating routine.
 * The pages this library follows describe no such variant: it exists only for these
 * callers.
 *
 * Formats: BONSAI_FMT_PTQ1_0 and BONSAI_FMT_PQ2_0 only; BONSAI_FMT_Q1_0 and
 * BONSAI_FMT_PQ2_0_G64 return BONSAI_ERR_FMT.
 * Limits: M must be 1, K a multiple of 512 and (K / 512) * N <= 1048576 (the array holds
 * 2^20 FP32 partials, 4 MiB, kept by every GPU that loads the library until the process
 * exits); other shapes return BONSAI_ERR_TOO_LARGE and launch nothing.  Checks run in
 * the order format, shape, NULL pointer, alignment, then these limits.  Inputs and
 * output are caller-owned device memory as for bonsai_ternary_linear.
 *
 * Set-up: the first call on each device looks up that device's copy of the array
 * (with that device current); make that first call before capturing any stream.
 * Every call shares the one array and leaves its partial sums there; each call writes
 * every partial it reads before reading it, so nothing needs clearing between calls.
 * Calls whose work overlaps on the GPU (different streams, or concurrent host threads)
 * race on the array -- serialise them. */
int bonsai_ternary_linear_noalloc(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                                  uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, void *stream);

/* Device status bits, set by a kernel whose bounded wait gave up (the call then wrote
 * NaN for the outputs it could not finish; see the conventions above).  They stay set
 * until cleared by bonsai_device_status. */
#define BONSAI_DEVICE_GEMV_COPY_TIMEOUT 1u  /* integer GEMV: a weight copy never landed      */
#define BONSAI_DEVICE_GEMV_PIECE_TIMEOUT 2u /* integer GEMV: a split tile's later piece, or  */
                                            /* its hand-over, never came                      */
#define BONSAI_DEVICE_GEMM_TIMEOUT 4u       /* prefill GEMM: a barrier or hand-over wait gave up */
#define BONSAI_DEVICE_SKINNY_TIMEOUT 8u     /* skinny kernel: the wait after the rotation   */
                                            /* phase, or a weight copy, never ended           */

/* Reads the calling device's status bits into *bits after synchronising `stream` (the
 * stream of the calls in question), and clears them when `clear` is non-zero.  *bits is 0
 * when no call has run on the device yet.  Returns BONSAI_ERR_NULL for a NULL bits,
 * BONSAI_ERR_CUDA if the copy or the synchronisation fails.  The pages describe no such
 * call; it reports the bounded waits of this implementation. */
int bonsai_device_status(void *stream, uint32_t *bits, int clear);

/* Test hook.  While enabled (enable != 0), the waits of the integer tensor-core GEMV for
 * the later pieces of its split row tiles, and of the prefill GEMM for its hand-over
 * flags, look for a call number that no CTA writes and give up after 64 polls: the calls
 * then write NaN for those tiles and set the status bits, without any fault, so that the
 * timeout path can be tested.  Off by default; applies to calls launched while enabled. */
int bonsai_debug_force_timeouts(int enable);

/* Frees the workspaces of every device (after synchronising each).  The
 * library stays usable: the next call allocates again. */
void bonsai_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* BONSAI_H */
