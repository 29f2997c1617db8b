/*
 * grinqh.h - C ABI of the GRINQH graded bit-plane VMM library (sm_100a).
 *
 * GRINQH ("GRINQH: Graded Input-based Quantization Hierarchy for Efficient LLM
 * Generation", arXiv 2606.23419) speeds up decoding by reading, for each
 * input channel k of a linear layer, only the b_k most significant bits of that
 * channel's b_max-bit weights (b_max = 8 by default; 2, 4 or 6 on request),
 * where b_k is chosen per token from |x_k| against calibrated thresholds
 * (Section 3.1), and b_k = 0 skips the channel entirely.
 * The weights are stored once, as MSB-first bit planes, so every narrower width
 * is a prefix of the wider one (Section 3.3, "Storage Layout and Weight
 * Loading").
 *
 * Calls, in the order a user makes them:
 *   grinqh_layout_init       sizes of the packed buffers for a K x N layer
 *                            (grinqh_layout_init_bmax for b_max < 8)
 *   grinqh_pack              offline b_max-bit RTN + bit-plane packing
 *   grinqh_maxent_distribution / grinqh_calibrate   thresholds for a target width
 *   grinqh_select            per-token grading + per-class channel lists
 *   grinqh_vmm               y = x . W_hat over the graded bit planes
 * and, for the same packed layer:
 *   grinqh_select_vmm        grading and the graded product in one launch
 *   grinqh_select_vmm_batch  the same for T tokens in one launch
 *   grinqh_select_vmm_batch_tc  the same on the tensor cores, one rebuild per row
 *   grinqh_vmm_noalloc       grinqh_vmm on the library's own static scratch
 *   grinqh_dequant / grinqh_prefill   full-width weights and the dense prefill
 *                            product for many tokens
 * and, for nested look-up-table codes (any-precision style):
 *   grinqh_lut_build         offline nested 2-means codes and tables (host)
 *   grinqh_pack_codes        bit planes of given b_max-bit codes
 *   grinqh_lut_bytes         size of the per-row table buffer
 *   grinqh_vmm_lut           y = x . W_hat with w_hat a table entry per width
 *
 * Conventions for every call:
 *   - W is K x N: K input channels (rows), N output channels (columns).
 *   - fp16 values are IEEE binary16 bit patterns passed as uint16_t.
 *   - "device" pointers are CUDA global-memory addresses of the current device;
 *     "host" pointers are ordinary CPU memory. The caller allocates and owns
 *     every buffer; the library never allocates, frees or synchronises
 *     (grinqh_prefill's cuBLAS handle is the one exception, see there).
 *   - stream is a cudaStream_t passed as void*; NULL means the legacy default
 *     stream. Every device call is asynchronous on that stream.
 *   - Arguments are checked on the host before anything is launched; a failed
 *     check returns an error code and launches nothing. A CUDA launch error is
 *     returned as GRINQH_ERR_CUDA. Nothing traps on the device.
 *   - Sizes: 1 <= K, N <= 2^24, K * N <= 2^34. Classes: 1..9 bit widths, strictly
 *     increasing, each in 0..8.
 */
#ifndef GRINQH_H_
#define GRINQH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GRINQH_GROUP 128       /* columns per (row, group) scale/zero pair */
#define GRINQH_MAX_CLASSES 9   /* widths 0..8 */
#define GRINQH_PLANES 8        /* largest b_max (the default) */

typedef enum {
  GRINQH_OK = 0,
  GRINQH_ERR_INVALID_ARG = 1,   /* a size, a pointer or a class set is invalid */
  GRINQH_ERR_ALIGNMENT = 2,     /* a pointer is not aligned as documented */
  GRINQH_ERR_UNSUPPORTED = 3,   /* valid, but outside what this build handles */
  GRINQH_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
  GRINQH_ERR_CUDA = 5           /* a CUDA runtime call failed */
} grinqh_status;

/*
 * Physical layout of a packed K x N layer. Filled by grinqh_layout_init or
 * grinqh_layout_init_bmax; treat as read-only. One device buffer (packed_bytes,
 * 16-byte aligned) holds the layer. Each row is cut into n_tiles column tiles
 * of tile_n = 1024 columns; row k, tile t is record r = k*n_tiles + t (a row's
 * tiles are adjacent). The buffer holds two arrays:
 *   planes   bytes [0, K*n_tiles*record_bytes): record r's planes at byte
 *            r*record_bytes, record_bytes = 128 * b_max (1024 for b_max = 8):
 *            the b_max bit planes of the b_max-bit codes, MSB first (plane
 *            p = 0 is bit b_max-1 of the code, p = b_max-1 is bit 0), in b_max/2
 *            plane pairs (the paper's 2-bit segments): pair s holds planes 2s
 *            and 2s+1 in bytes [256s, 256(s+1)) of the record;
 *   scale/zero  bytes [K*n_tiles*record_bytes, packed_bytes): 32 bytes per
 *            record, record r's at r*32 from the start of the array: 8 uint32
 *            words, word g = scale_fp16 | (zero_fp16 << 16) of columns
 *            [t*1024 + 128g, +128) (0 past the last group).
 * So the top b planes of a (row, tile) are one contiguous, 256-byte-aligned run
 * of 256 ceil(b/2) bytes (for odd b the last pair's second plane is read and
 * not used), and its scale/zero words one 32-byte sector: no DRAM sector holds
 * bytes of two records. Inside pair s, 32-bit word 2w holds local columns
 * 32w..32w+15 and word 2w+1 columns 32w+16..32w+31; in either word, column
 * 4j' + i of that half (j' in 0..3, i in 0..3) of plane 2s + l sits at bit
 * (8i + 2j' + 7 - 2s - l) mod 32. Columns >= N are zero bits.
 */
typedef struct {
  int32_t K;             /* input channels (rows) */
  int32_t N;             /* output channels (columns) */
  int32_t n_groups;      /* ceil(N / 128) */
  int32_t tile_n;        /* columns per tile (1024) */
  int32_t n_tiles;       /* ceil(N / tile_n) */
  int32_t record_bytes;  /* plane bytes per (row, tile) record: 128 * b_max */
  int32_t b_max;         /* bits per stored code: 2, 4, 6 or 8 */
  int32_t reserved;      /* 0 */
  int64_t packed_bytes;  /* K * n_tiles * (record_bytes + 32): planes, then scale/zero words */
} grinqh_layout;

/* Library version string (static storage). */
const char* grinqh_version(void);

/* Human-readable name of a status code (static storage). */
const char* grinqh_status_string(grinqh_status s);

/*
 * Fill *out with the packed layout of a K x N layer of 8-bit codes. Host only.
 * Errors: INVALID_ARG for out == NULL or sizes outside the limits above.
 */
grinqh_status grinqh_layout_init(int32_t K, int32_t N, grinqh_layout* out);

/*
 * The same for codes of b_max bits. Paper: Section 3.3 (every weight becomes
 * one b_max-bit integer kept as 2-bit segments, so that any even width
 * b in {0, 2, ..., b_max} can be fetched; the evaluation uses b_max in {4, 6, 8}).
 * This library takes any width 0..b_max (1-bit planes in pairs) and
 * b_max in {2, 4, 6, 8}; grinqh_layout_init(K, N, out) is b_max = 8. Host only.
 * Errors: INVALID_ARG for out == NULL, sizes outside the limits above or b_max
 * not in {2, 4, 6, 8}.
 */
grinqh_status grinqh_layout_init_bmax(int32_t K, int32_t N, int32_t b_max, grinqh_layout* out);

/*
 * Offline b_max-bit RTN quantisation and bit-plane packing (b_max from the
 * layout, L = 2^b_max - 1 levels; L = 255 for the default b_max = 8).
 * Paper: Section 3.3 (uniform b_max-bit quantisation, nested slices, input-major
 * storage), Section 4 (RTN, group size G = 128), Appendix C.1 (same-significance
 * bits of neighbouring weights packed into 32-bit words).
 * Per (row k, group g): s = fp16_rne((max - min) / L) computed in fp64 and
 * rounded straight to fp16 (s := 1 if it rounds to 0, s := 65504 if it
 * overflows); z = clamp(rne(-min / s), 0, L); q = clamp(rne(w / s) + z, 0, L),
 * quotients in fp64, ties to even.
 *   W       device, fp32 [K][N] row-major, finite values (non-finite input
 *           gives unspecified codes), 4-byte aligned.
 *   packed  device, layout->packed_bytes, 16-byte aligned; fully overwritten.
 * Errors: INVALID_ARG (NULL pointers, layout inconsistent), ALIGNMENT, CUDA.
 */
grinqh_status grinqh_pack(const grinqh_layout* layout, const float* W, void* packed, void* stream);

/*
 * Decode the codes the VMM uses, for testing the packed format. For each row k
 * with width b = bits[k] (b_max for every row when bits == NULL):
 *   b = 0: code 0 (the row is never read by grinqh_vmm);
 *   1 <= b < b_max: c_b * 2^(b_max-b) + 2^(b_max-b-1), c_b = top b bits of the
 *     b_max-bit code q (Section 3.3 reconstruction with its midpoint term);
 *   b = b_max: q.
 *   packed  device, as written by grinqh_pack for the same layout.
 *   bits    device uint8 [K] of widths 0..b_max (a larger width decodes as
 *           b_max), or NULL.
 *   codes   device uint8 [K][N] row-major; fully overwritten.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA.
 */
grinqh_status grinqh_unpack_codes(const grinqh_layout* layout, const void* packed,
                                  const uint8_t* bits, uint8_t* codes, void* stream);

/*
 * Full-width dequantisation (the first step of the prefill path).
 * Paper: Section 4, "Prefill vs. Decoding Evaluation" (prefill unpacks the
 * weights at full b_max precision for a dense product) and Section 3.3
 * (w_hat = s * (q - z) at b = b_max). W16[k][n] = w_hat rounded once to binary16
 * (round to nearest even; the product itself is exact).
 *   packed  device, from grinqh_pack with this layout, 16-byte aligned.
 *   W16     device binary16 [K][N] row-major, 16-byte aligned; fully overwritten.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA.
 */
grinqh_status grinqh_dequant(const grinqh_layout* layout, const void* packed, uint16_t* W16, void* stream);

/*
 * The prefill product: Y = X . W_hat for T tokens at full width (no grading),
 * as grinqh_dequant into W16 followed by a dense binary16 GEMM with fp32
 * accumulation (cuBLAS, on the same stream). Paper: Section 4, "Prefill vs.
 * Decoding Evaluation". This call links cuBLAS, which allocates its handle's
 * resources the first time a device uses it; call it once before any stream
 * capture.
 *   X     device fp16 [T][K] row-major, 2-byte aligned; 1 <= T <= 2^24.
 *   Y     device fp32 [T][N] row-major, output (overwritten), 4-byte aligned.
 *   W16   device binary16 [K][N], 16-byte aligned: scratch that receives the
 *         dequantised weights (and keeps them after the call).
 * Errors: INVALID_ARG, ALIGNMENT, CUDA.
 */
grinqh_status grinqh_prefill(const grinqh_layout* layout, const void* packed, const uint16_t* X, int32_t T,
                             float* Y, uint16_t* W16, void* stream);

/*
 * The prefill product fused on the tensor cores: the same Y = X . W_hat (same
 * binary16 operands w_hat = fp16_rne(s (q - z)) as grinqh_dequant, fp32
 * accumulation) without writing W_hat to memory: each CTA rebuilds a 128-column
 * slice of W_hat from the bit planes into shared memory, 64 rows at a time, and
 * the 5th-generation tensor cores (tcgen05, sm_100a) multiply it with TMA-loaded
 * tiles of 256 or 512 tokens (K split over a cluster of 2 or 4 CTAs when the
 * grid is small), accumulating in tensor memory. Paper: Section 4,
 * "Prefill vs. Decoding Evaluation" (full b_max precision, dense product) and
 * Section 5 (unpacking fused with the product). Allocates nothing and links no
 * library kernel; the summation order differs from grinqh_prefill's, so the two
 * agree within the tolerance, not bitwise.
 *   X       device fp16 [T][K] row-major, 16-byte aligned; K a multiple of 8;
 *           1 <= T <= 65535 * 256.
 *   Y       device fp32 [T][N] row-major, output (overwritten), 4-byte aligned.
 *   status  device, 16 bytes, 16-byte aligned, zero-filled before first use;
 *           bit 0 of its first word is set if a wait inside the kernel gave up
 *           after about a second (Y is then invalid); no call clears it.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (K not a multiple of 8, T above the
 * limit), CUDA.
 */
grinqh_status grinqh_prefill_tc(const grinqh_layout* layout, const void* packed, const uint16_t* X, int32_t T,
                                float* Y, uint32_t* status, void* stream);

/*
 * Nested look-up-table codes. Paper: Section 3.3 ("Storage Layout and Weight
 * Loading": the planes need a nested quantisation, met by uniform codes and by
 * k-means codes such as any-precision LLM's; with such tables no midpoint term
 * is used, the nested levels being centred already), Section 4 ("Models and
 * Baselines": any-precision LLM weights at b_max = 8) and Appendix E.2.
 * Library reading: each row k has one table per width b = 1..b_max; the top b
 * bits c_b = q >> (b_max - b) of a b_max-bit code q select its entry, and
 * w_hat = T_k[2^b + c_b]. The tables of a row are stored in heap order as
 * binary16: entry 2^b + c is entry c of width b, entries 0 and 1 are never read,
 * so a row holds 2^(b_max+1) entries (2^(b_max+2) bytes, 1 KB at b_max = 8).
 */

/*
 * Bit planes of caller-given codes: the packed layout of grinqh_layout_init_bmax
 * with every record's scale/zero words zero and the planes of codes[k][n] (only
 * its low b_max bits are used). Columns >= N are zero bits.
 *   codes   device uint8 [K][N] row-major, any alignment.
 *   packed  device, packed_bytes, 16-byte aligned, fully overwritten.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA.
 */
grinqh_status grinqh_pack_codes(const grinqh_layout* layout, const uint8_t* codes, void* packed, void* stream);

/*
 * Offline construction of nested table codes on the host (no CUDA): any-precision
 * style incremental upscaling (Appendix E.2). For each row, width 0 is one
 * cluster; every cluster of width b - 1 is cut in two at the optimal 1-D 2-means
 * point of its sorted members (never between equal values; the smallest cut on a
 * tie; the lower half gets bit 0; a cluster with fewer than two distinct values
 * keeps all members in its lower half, and an empty half takes its parent's
 * value). Entry c of width b is its members' mean, rounded once to binary16, at
 * heap index 2^b + c (entry 0 is 0, entry 1 the row mean); a weight's code is
 * its cluster at width b_max. Unweighted (the pages' seed model and sensitivity
 * weights need trained models). Cost O(K N (log N + b_max)).
 *   W      host fp32 [K][N] row-major, finite.
 *   codes  host uint8 [K][N] row-major, output (b_max-bit codes for grinqh_pack_codes).
 *   lut    host binary16 [K][2^(b_max+1)], output (the tables of grinqh_vmm_lut).
 * Errors: INVALID_ARG (sizes, b_max not in {2, 4, 6, 8}, NULL, non-finite W).
 */
grinqh_status grinqh_lut_build(const float* W, int32_t K, int32_t N, int32_t b_max, uint8_t* codes, uint16_t* lut);

/* Bytes of the table buffer of grinqh_vmm_lut: K * 2^(b_max+2). */
grinqh_status grinqh_lut_bytes(const grinqh_layout* layout, size_t* bytes);

/*
 * y = x . W_hat over nested table codes, graded as grinqh_vmm: for a channel of
 * width b_k > 0, w_hat[k][n] = lut[k][2^b_k + (q[k][n] >> (b_max - b_k))]; rows of
 * width 0 are not read. Reads only the top b_k planes of row k (not its
 * scale/zero words) and the b_k-bit part of row k's table.
 *   packed     device, from grinqh_pack_codes (or grinqh_pack: its codes are
 *              then read as table indices), 16-byte aligned.
 *   lut        device binary16 [K][2^(b_max+1)] in heap order, 16-byte aligned.
 *   x, idx, offsets, classes, n_classes, y, workspace, workspace_bytes: as for
 *              grinqh_vmm (the same selection and the same workspace size).
 * Errors: INVALID_ARG (also a class wider than b_max), ALIGNMENT, WORKSPACE, CUDA.
 */
grinqh_status grinqh_vmm_lut(const grinqh_layout* layout, const void* packed, const uint16_t* lut,
                             const uint16_t* x, const int32_t* idx, const int32_t* offsets, const uint8_t* classes,
                             int32_t n_classes, float* y, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Maximum-entropy precision distribution P over a class set for a requested
 * mean width target_bits (host only, no CUDA). Paper: Appendix A.1 eq. (1)
 * constrains P to the simplex with sum_i p_i b_i = b*; the objective there is a
 * model-quality metric, which needs trained models. This library takes the
 * distribution of maximum entropy, p_i proportional to exp(lambda * b_i), with
 * lambda found by fp64 bisection. target_bits equal to the smallest or largest
 * class gives the one-hot distribution of that class.
 *   classes  host uint8 [n_classes], strictly increasing widths in 0..8.
 *   P        host double [n_classes], output.
 * Errors: INVALID_ARG (bad class set, target outside [classes[0],
 * classes[n_classes-1]], NULL pointers).
 */
grinqh_status grinqh_maxent_distribution(const uint8_t* classes, int32_t n_classes,
                                         double target_bits, double* P);

/* Workspace bytes grinqh_calibrate needs for S samples and n_classes classes. */
grinqh_status grinqh_calibrate_workspace_bytes(int32_t S, int32_t n_classes, size_t* bytes);

/*
 * Threshold calibration by percentile mapping. Paper: Section 3.2 and Appendix
 * A.1 eq. (2): for every calibration sample, theta_j is the
 * (p_0 + ... + p_{j-1})-quantile of |x|; the per-sample values are averaged.
 * Readings used here: n_classes - 1 thresholds; quantile = linear interpolation
 * at position q_j*(K-1) of the ascending magnitudes (fp64); mean over samples
 * summed in ascending sample order in fp64, then rounded to fp32; theta_j = 0
 * when q_j == 0 exactly; theta_j = +inf when p_j..p_n are all zero.
 *   X           device, fp16 [S][K] calibration vectors, finite, 2-byte aligned.
 *   classes     host uint8 [n_classes].
 *   P           host double [n_classes] (each >= 0, sum 1 within 1e-9), or NULL
 *               to use grinqh_maxent_distribution(classes, target_bits).
 *   thresholds  device fp32 [n_classes - 1], output, 4-byte aligned.
 *   workspace   device, >= grinqh_calibrate_workspace_bytes, 16-byte aligned.
 * Limits: 1 <= S <= 65535, 1 <= K <= 2^24.
 * Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, CUDA.
 */
grinqh_status grinqh_calibrate(const uint16_t* X, int32_t S, int32_t K, const uint8_t* classes,
                               int32_t n_classes, const double* P, double target_bits,
                               float* thresholds, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * Per-token grading and stable per-class compaction.
 * Paper: Section 3.1: channel k gets class j = #{ i : |x_k| >= theta_i } (the
 * interval rule [theta_j, theta_{j+1}) with theta_0 = 0, theta_{n+1} = inf,
 * written as a count so that ties go to the upper class); NaN goes to class 0.
 *   x          device fp16 [K].
 *   thresholds device fp32 [n_classes - 1].
 *   classes    host uint8 [n_classes].
 *   bits       device uint8 [K], output: classes[j_k].
 *   idx        device int32 [K], output: channel indices, class-major, ascending
 *              k inside each class.
 *   offsets    device int32 [n_classes + 1], output: offsets[j] = first position
 *              of class j in idx, offsets[n_classes] = K.
 * All device pointers 4-byte aligned except x (2) and bits (1).
 * Limits: 1 <= K <= 65536. Every block of 1024 channels reads all of x (from
 * L2) to count the channels of each class ahead of it, so one call reads
 * K^2 / 512 bytes from L2: 8 MiB at K = 65536, more than every linear of the
 * evaluated models needs. For larger K the call returns UNSUPPORTED; callers
 * with such layers build idx and offsets themselves for grinqh_vmm.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (K > 65536), CUDA.
 */
grinqh_status grinqh_select(const uint16_t* x, int32_t K, const float* thresholds,
                            const uint8_t* classes, int32_t n_classes, uint8_t* bits,
                            int32_t* idx, int32_t* offsets, void* stream);

/* Workspace bytes grinqh_vmm needs for a layout. */
grinqh_status grinqh_vmm_workspace_bytes(const grinqh_layout* layout, size_t* bytes);

/*
 * The graded vector-matrix product (the decode hot path).
 * Paper: Fig. 2 and Section 3.3: for every channel k with b_k > 0, only planes
 * 0..b_k-1 of row k (and its scale/zero words) are read; the row is rebuilt as
 * w_hat = s * (code - z) with code = c_b * 2^(b_max-b) + 2^(b_max-b-1) for
 * b < b_max and q for b = b_max (b_max = 8 unless the layout says otherwise);
 * channels with b_k = 0 are never read and add nothing.
 *   y[n] = sum_k x_k * w_hat[k][n], accumulated in fp32.
 *   packed        device, from grinqh_pack with this layout.
 *   x             device fp16 [K] (the same vector grinqh_select graded).
 *   idx, offsets  device, from grinqh_select with the same classes.
 *   classes       host uint8 [n_classes]; every width at most the layout's
 *                 b_max (INVALID_ARG otherwise).
 *   y             device fp32 [N], output (overwritten), 4-byte aligned.
 *   workspace     device, >= grinqh_vmm_workspace_bytes(layout) (a size that
 *                 depends on the current device's SM count), 16-byte aligned;
 *                 its first 16 bytes must be zero-filled once before first use.
 *                 They hold a status word that stays 0 (reserved: the kernels
 *                 of this version contain no wait that can time out; a nonzero
 *                 word would mean the call's output is invalid). The rest holds
 *                 per-CTA partial sums of y, fully rewritten by every call.
 *                 Calls that share a workspace must not overlap in time.
 * y is written with plain stores in a fixed summation order, so repeated calls
 * on the same inputs give bitwise identical results.
 * Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, CUDA.
 */
grinqh_status grinqh_vmm(const grinqh_layout* layout, const void* packed,
                         const uint16_t* x, const int32_t* idx, const int32_t* offsets,
                         const uint8_t* classes, int32_t n_classes, float* y, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * Grading and the graded product in one call: y = x . W_hat over the same
 * graded rows as grinqh_select followed by grinqh_vmm (every channel gets the
 * class and width grinqh_select gives it), without the channel lists in
 * memory. The rows are summed in another order than grinqh_vmm's, so the two
 * agree within fp32 rounding (both meet the same error bound), not bitwise;
 * repeated calls on the same inputs give bitwise identical results.
 * Paper: Section 3.1 (grading, "Dynamic Precision Assignment"), Fig. 2 and
 * Section 3.3 (the graded product); the fusion is this library's: the CTAs of
 * row split r grade the channels k = r, r + R, r + 2R, ... themselves and read
 * the rows of those with nonzero width, so no selection kernel, no kernel
 * boundary and no channel-list read precede the weights.
 *   packed, classes, y, workspace, workspace_bytes   as grinqh_vmm (the same
 *                workspace size, grinqh_vmm_workspace_bytes).
 *   x            device fp16 [K], 2-byte aligned.
 *   thresholds   device fp32 [n_classes - 1], 4-byte aligned (NULL allowed
 *                when n_classes == 1); any order, NaN never reached.
 * Limit: K <= 16384 (GRINQH_ERR_UNSUPPORTED above; use grinqh_select and
 * grinqh_vmm there).
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, WORKSPACE, CUDA.
 */
grinqh_status grinqh_select_vmm(const grinqh_layout* layout, const void* packed, const uint16_t* x,
                                const float* thresholds, const uint8_t* classes, int32_t n_classes,
                                float* y, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes grinqh_select_vmm_batch needs for a layout and a token count. */
grinqh_status grinqh_vmm_batch_workspace_bytes(const grinqh_layout* layout, int32_t tokens, size_t* bytes);

/*
 * grinqh_select_vmm for a batch of tokens in one launch: row t of Y is exactly
 * what grinqh_select_vmm gives for row t of X (the same bits). Paper: Section
 * 3.1 (every token grades every channel from its own |x|) and Section 6, which
 * states that the method targets batch size one; this library's reading for a
 * batch keeps every token's grading and reconstruction as at batch one. The
 * tokens' CTAs run one token after another on the same weights, so a row that
 * several tokens need is read from DRAM about once (the union of the tokens'
 * widths) and from L2 after that, as long as the layer's graded bytes fit in L2.
 *   X            device fp16 [tokens][K] row-major, 2-byte aligned.
 *   tokens       1..65535.
 *   Y            device fp32 [tokens][N] row-major, output (overwritten).
 *   thresholds   as grinqh_select_vmm (shared by every token).
 *   workspace    device, >= grinqh_vmm_batch_workspace_bytes(layout, tokens),
 *                16-byte aligned, first 16 bytes zero-filled once before first use.
 * Limit: K <= 16384 (GRINQH_ERR_UNSUPPORTED above).
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, WORKSPACE, CUDA.
 */
grinqh_status grinqh_select_vmm_batch(const grinqh_layout* layout, const void* packed, const uint16_t* X,
                                      int32_t tokens, const float* thresholds, const uint8_t* classes,
                                      int32_t n_classes, float* Y, void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * The batched graded product on the 5th-generation tensor cores: Y[t] = the graded
 * product of X[t] (every token graded from its own |x| and every row rebuilt at
 * that token's width, as grinqh_select_vmm does), with each row's planes read
 * and merged once for all tokens. Paper: Section 3.1 (per-token grading), Section
 * 3.3 (nested codes and bin midpoints) and Section 6 (the method targets batch
 * size one; this library keeps every token's grading). Per 128-column group the
 * product is split by width class into tcgen05 MMAs (sm_100a): the codes masked
 * to the class's width times a power of two (exact in binary16) against x times
 * the scale's significand split into two binary16 parts, fp32 accumulation; the
 * bin midpoint and zero point enter as a per-token constant in fp32. Results
 * agree with grinqh_select_vmm_batch within the VMM tolerance, not bitwise.
 * Deterministic: the same inputs give the same bits. Allocates nothing.
 *   X        device fp16 [tokens][K] row-major, 16-byte aligned; K a multiple of 8.
 *   tokens   1..65535; CTAs take 32 tokens each.
 *   thresholds, classes, n_classes: as grinqh_select_vmm.
 *   Y        device fp32 [tokens][N], output (overwritten), 4-byte aligned.
 *   status   device, 16 bytes, 16-byte aligned, zero-filled before first use;
 *            bit 0 of its first word: a wait inside the kernel gave up after about
 *            a second; bit 1: a value outside the binary16 range of the operands
 *            (|x| times the scale's significand, rounded to binary16, of 32768 or
 *            more, or a scale of 2^(14 - b_max) or more). Either bit means Y is
 *            not valid; no call clears them.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (K not a multiple of 8), CUDA.
 */
grinqh_status grinqh_select_vmm_batch_tc(const grinqh_layout* layout, const void* packed, const uint16_t* X,
                                         int32_t tokens, const float* thresholds, const uint8_t* classes,
                                         int32_t n_classes, float* Y, uint32_t* status, void* stream);

/*
 * grinqh_vmm without a caller-provided workspace. The paper has no counterpart:
 * this is a calling convention of the library, not a step of the method.
 * It computes exactly what grinqh_vmm computes (same kernels, same summation
 * order, so the same bits of y) but takes its scratch (status word and per-CTA
 * partial sums) from one static device array of 1 MiB inside the library,
 * and allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 * routine. It is for callers that have no device allocator to hand a workspace
 * from: a plain C host that links only this library and the CUDA runtime, or a
 * process that reserves all device memory up front for a fixed pool, where an
 * allocation at call time could fail or fragment the pool.
 *   Arguments as grinqh_vmm, without workspace and workspace_bytes.
 * The scratch is shared by every call on a device: calls of this entry point
 * that overlap on the GPU (e.g. on two streams at once) race on it and give
 * undefined y. Its 16-byte status word starts at zero when the library's
 * device code is loaded and stays zero in this version; the partial sums need
 * no clearing.
 * Limit: a layout whose grinqh_vmm_workspace_bytes exceeds 1 MiB is rejected
 * with GRINQH_ERR_WORKSPACE (on a 148-SM B200 every layout fits: at most 148
 * row splits x column tiles of 4 KiB each).
 * Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, CUDA.
 */
grinqh_status grinqh_vmm_noalloc(const grinqh_layout* layout, const void* packed,
                                 const uint16_t* x, const int32_t* idx, const int32_t* offsets,
                                 const uint8_t* classes, int32_t n_classes, float* y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GRINQH_H_ */
