/*
 * dbc.h -- C ABI of the B200 dynamic byte-chunking library (libdbc.so).
 *
 * The library implements the chunking stage of hierarchical byte models:
 *   - ByteFlow's coding-rate downsampler (arXiv 2603.03583): the marginal
 *     lossy coding rate dR_t of every byte position, Top-K boundary selection
 *     with the first position fixed, the gather of the chunk vectors (with an
 *     optional local->global projection) and the 16-bin multi-linear upsampler
 *     with its residual;
 *   - an H-Net style cosine-similarity router with EMA smoothing, as a second
 *     boundary rule (ByteGen analysis report, "H-Net architecture").
 *
 * Conventions shared by every entry point
 *   - All pointers named H, dR, idx, Z, S, p, ... are DEVICE pointers owned by
 *     the caller; the library never allocates device memory.  Calls that need
 *     scratch take a caller-provided workspace `ws` of at least the size that
 *     the matching *_workspace() query returns (256-byte aligned).
 *   - Every call is asynchronous on `stream` (0 = legacy default stream), does
 *     not synchronise the host and returns a dbc_status.  Argument errors are
 *     detected on the host and returned before anything is launched.
 *   - Errors found on the device (non-finite input, bound violations) are
 *     OR-ed as bit flags (1 << code) into `*dev_status` when that pointer is
 *     non-NULL; the caller reads it after synchronising.  Kernels never trap.
 *   - Positions are 0-based.  A batch holds `rows` sequences packed back to
 *     back: with `offsets == NULL` the batch is dense (row r covers positions
 *     [r*T, (r+1)*T)); otherwise `offsets` is a device int64 array of rows+1
 *     non-decreasing entries with offsets[0] = 0 and offsets[rows] = N (ragged
 *     batch, rows may be empty; `T` is then an upper bound of the row length).
 *   - Features are row-major [N, d].  `dtype` says whether H holds fp32 or
 *     bf16 values.  Supported feature widths: d in {64, 128, 256, 512}.
 */
#ifndef DBC_H_
#define DBC_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DBC_API __attribute__((visibility("default")))
#else
#define DBC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *dbc_stream_t;   /* same type as cudaStream_t */

typedef enum {
    DBC_OK = 0,
    DBC_ERR_INVALID_ARG = 1,   /* NULL pointer, bad size, misalignment, K < 1, eps2 <= 0 */
    DBC_ERR_UNSUPPORTED = 2,   /* feature width or dtype not supported */
    DBC_ERR_CUDA = 3,          /* a CUDA launch/runtime call failed */
    DBC_ERR_NONFINITE = 4,     /* device: NaN/Inf met in an input (flag only) */
    DBC_ERR_TIMEOUT = 5,       /* device: a bounded wait gave up (flag only) */
    DBC_ERR_BOUNDS = 6,        /* device: an index left its valid range (flag only) */
    DBC_ERR_WORKSPACE = 7      /* workspace NULL or smaller than required */
} dbc_status;

typedef enum { DBC_F32 = 0, DBC_BF16 = 1 } dbc_dtype;

/* Bin rules of the upsampler (the pages disagree; see each entry). */
typedef enum {
    DBC_BIN_IN_CHUNK_OFFSET = 0,    /* b = min(t - s_c, nbins - 1)       (default) */
    DBC_BIN_IN_CHUNK_FRACTION = 1,  /* b = floor(nbins (t - s_c) / L_c)            */
    DBC_BIN_ABSOLUTE = 2            /* b = floor(t nbins / T_row)                   */
} dbc_bin_mode;

/* Human-readable name of a status code (static storage). */
DBC_API const char *dbc_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
DBC_API int dbc_version(void);

/* Number of CUDA kernels launched by this library in this process so far
 * (all entry points, all host threads); a profiling aid. */
DBC_API uint64_t dbc_launch_count(void);

/* -------------------------------------------------------------------------
 * chunk_coding_rate -- marginal lossy coding rate of every position.
 *
 * ByteFlow (paper.rainbus.top summary, "Prerequisites: lossy coding rate" and
 * "Method steps", stage 2; papernotes.org notes, "Key design 2"):
 *   R_eps(H) = 1/2 logdet(I + c H H^T),  c = d / eps2,
 *   dR_t = R_eps(h_{0..t}) - R_eps(h_{0..t-1})   for each row separately,
 * with R of the empty prefix = 0.  Computed through the identity
 *   dR_t = 1/2 log(1 + c h_t^T M_{t-1}^{-1} h_t),  M_t = I_d + c sum_{i<=t} h_i h_i^T.
 *
 * H       [N, d] fp32 or bf16 (dtype), 16-byte aligned.
 * offsets NULL (dense, N = rows*T) or int64 [rows+1] (ragged).
 * rows, T rows >= 0; T = row length (dense) or an upper bound (ragged).
 * N       total positions (must equal rows*T when dense).
 * eps2    eps^2 > 0.
 * dR      out, fp32 [N].
 * ws      workspace of chunk_coding_rate_workspace(rows, T, N, d) bytes.
 * Errors: INVALID_ARG (NULL/negative/misaligned/eps2 <= 0/N mismatch),
 *         UNSUPPORTED (d or dtype), WORKSPACE, CUDA; device flag NONFINITE.
 * ------------------------------------------------------------------------- */
DBC_API size_t chunk_coding_rate_workspace(int64_t rows, int64_t T, int64_t N, int64_t d);
DBC_API dbc_status chunk_coding_rate(const void *H, int dtype, const int64_t *offsets,
                             int64_t rows, int64_t T, int64_t N, int64_t d,
                             float eps2, float *dR, void *ws, size_t ws_bytes,
                             int32_t *dev_status, dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * chunk_coding_rate_stream -- the marginal coding rate of streams delivered in
 * blocks (causal use of the chunker).
 *
 * ByteFlow (summary "Prerequisites: lossy coding rate" and "Method steps",
 * stage 2; notes "Key design 2"): dR_t = R(h_{0..t}) - R(h_{0..t-1}).  A
 * stream that has already consumed t0 positions carries the Gram sum
 * S = sum_{i < t0} h_i h_i^T of everything seen; the next n positions' dR are
 * the whole sequence's values at t0 .. t0 + n - 1 (same definition, same
 * segment boundaries 0, 64, 128, 256, 512, ... counted from the stream's start),
 * and S is advanced by the block.  Selecting boundaries causally is left to
 * the caller, e.g. chunk_topk_select over fixed windows of the stream.
 *
 * H        bf16 [streams, n, d] the new positions (d = 256 only).
 * t0       positions each stream consumed before this call (all streams
 *          equal); 0 starts the streams (state must then be zero).
 * state    in/out float64 [streams, d, d]: S before the call, S after it.
 *          Caller-owned, 16-byte aligned; zero it once per new stream.
 * dR       out fp32 [streams, n].
 * ws       workspace of chunk_coding_rate_stream_workspace(streams, n, t0, d)
 *          bytes (it depends on t0 through the segment cut).
 * Errors: INVALID_ARG, UNSUPPORTED (dtype other than bf16, d != 256),
 * WORKSPACE, CUDA; device flags NONFINITE, TIMEOUT.
 * ------------------------------------------------------------------------- */
DBC_API size_t chunk_coding_rate_stream_workspace(int64_t streams, int64_t n, int64_t t0, int64_t d);
DBC_API dbc_status chunk_coding_rate_stream(const void *H, int dtype, int64_t streams, int64_t n, int64_t d,
                                            int64_t t0, float eps2, double *state, float *dR, void *ws,
                                            size_t ws_bytes, int32_t *dev_status, dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * chunk_coding_rate_step -- the marginal coding rate of streams, one new
 * position at a time (the per-byte recursion).
 *
 * ByteFlow (summary "Prerequisites: lossy coding rate", "Method steps",
 * stage 2, "Limitations and improvements" first point, and "Weaknesses of the
 * independent analysis": an incremental per-byte update).  Each stream
 * carries B = L^{-T}, the inverse transposed Cholesky factor of
 * M = I + c sum h_i h_i^T over everything it has seen (c = d / eps2).  For
 * each new position h, in order: w = sqrt(c) B^T h, dR = 1/2 log(1 + |w|^2),
 * and B becomes the factor of M + c h h^T (an O(d^2) rank-one update of B).
 * The values equal the whole sequence's dR (same definition as
 * chunk_coding_rate) up to fp32 rounding, for any split of the stream into
 * calls; a call costs O(n d^2) on one SM per stream, so long blocks are
 * cheaper through chunk_coding_rate_stream.
 *
 * H        fp32 or bf16 (dtype) [streams, n, d] the new positions; d a
 *          multiple of 4, at most 256.
 * B_state  in/out fp32 [streams, d, d] row-major, 16-byte aligned: the upper
 *          triangle (with the diagonal) holds B before and after the call; the
 *          strictly lower triangle is not used and keeps its values (rows move
 *          in 16-byte pieces, so up to three entries left of each diagonal are
 *          read and written back unchanged).  A new stream starts from the
 *          identity (M = I).  Caller-owned; not to be written by other work
 *          while the call runs.
 * dR       out fp32 [streams, n].
 * Errors: INVALID_ARG (NULL, negative sizes, eps2 <= 0, misaligned state),
 * UNSUPPORTED (dtype, d > 256 or not a multiple of 4), CUDA; device flag
 * NONFINITE.
 * ------------------------------------------------------------------------- */
DBC_API dbc_status chunk_coding_rate_step(const void *H, int dtype, int64_t streams, int64_t n, int64_t d,
                                          float eps2, float *B_state, float *dR, int32_t *dev_status,
                                          dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * chunk_topk_select -- boundary positions per row.
 *
 * ByteFlow (notes "Key design 2"; summary stage 2): position 0 (BOS) is always
 * kept; the K-1 positions with the largest dR among t >= 1 are added; the K
 * boundaries are returned in increasing position.  Equal dR values are taken
 * in increasing position.  A row of length T_r yields min(K_r, T_r) indices.
 *
 * dR        fp32 [N].
 * offsets   NULL (dense) or int64 [rows+1].
 * K_per_row NULL, or device int64 [rows] giving K_r (each >= 1); when NULL,
 *           every row uses K_scalar (>= 1).
 * idx       out, int64, row-relative positions, rows stacked; capacity must be
 *           >= sum_r min(K_r, T_r) (rows*min(K_scalar,T) when dense).
 * idx_offsets out, int64 [rows+1]: row r's indices are idx[idx_offsets[r] ..
 *           idx_offsets[r+1]).
 * ws        workspace of chunk_topk_select_workspace(rows) bytes.
 * Errors: INVALID_ARG, WORKSPACE, CUDA; device flags NONFINITE (NaN in dR),
 *         BOUNDS (a K_r < 1).
 * ------------------------------------------------------------------------- */
DBC_API size_t chunk_topk_select_workspace(int64_t rows);
DBC_API dbc_status chunk_topk_select(const float *dR, const int64_t *offsets, int64_t rows,
                             int64_t T, int64_t N, const int64_t *K_per_row,
                             int64_t K_scalar, int64_t *idx, int64_t *idx_offsets,
                             void *ws, size_t ws_bytes, int32_t *dev_status,
                             dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * chunk_gather -- chunk vectors z_k = h_{s_k} (ByteFlow summary, stage 2),
 * optionally followed by the local->global projection z_k W_proj.
 *
 * H        [N, d] (dtype); offsets NULL (dense, row length T) or int64 [rows+1].
 * idx, idx_offsets as produced by chunk_topk_select; total_K = idx_offsets[rows].
 * Z        out, [total_K, d] same dtype as H: a bit-exact copy of the rows.
 * W_proj   NULL, or bf16 [d, d_g] (requires dtype == DBC_BF16); then
 *          Zp_f32 (fp32 [total_K, d_g], may be NULL) and Zp_bf16 (bf16, RNE of
 *          the fp32 result, may be NULL) receive Z W_proj with fp32 accumulation.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA; device flag BOUNDS (idx out of row).
 * ------------------------------------------------------------------------- */
DBC_API dbc_status chunk_gather(const void *H, int dtype, const int64_t *offsets, int64_t T,
                        int64_t d, const int64_t *idx, const int64_t *idx_offsets,
                        int64_t rows, int64_t total_K, void *Z, const void *W_proj,
                        int64_t d_g, float *Zp_f32, void *Zp_bf16,
                        int32_t *dev_status, dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * chunk_upsample -- multi-linear upsampling with residual.
 *
 * ByteFlow (summary stage 4; notes "Key design 4"): for each position t of a
 * row, c(t) = max{k : s_k <= t}, b(t) by `mode`, and
 *   S_t = h_t + g_{c(t)} W_{b(t)}.
 *
 * G        bf16 [total_K, d_g] chunk vectors (rows stacked like idx).
 * H        [N, d_l] (dtype) residual input; offsets NULL (dense) or int64 [rows+1].
 * idx, idx_offsets boundaries (each row's first index must be 0, increasing).
 * W_bin    bf16 [nbins, d_g, d_l] row-major; nbins in [1, 64].
 * S        out, fp32 [N, d_l].
 * ws       workspace of chunk_upsample_workspace(rows, N, nbins) bytes.
 * Supported: d_g, d_l multiples of 64 up to 2048.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA; device flag BOUNDS.
 * ------------------------------------------------------------------------- */
DBC_API size_t chunk_upsample_workspace(int64_t rows, int64_t N, int nbins);
DBC_API dbc_status chunk_upsample(const void *G, int64_t d_g, const void *H, int dtype,
                          const int64_t *offsets, int64_t T, int64_t N, int64_t d_l,
                          const int64_t *idx, const int64_t *idx_offsets, int64_t rows,
                          const void *W_bin, int nbins, int mode, float *S,
                          void *ws, size_t ws_bytes, int32_t *dev_status,
                          dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * chunk_upsample_backward -- gradients of the upsampling (for training).
 *
 * ByteFlow (summary stage 4; notes "Key design 4"), differentiated: with
 * dS = dL/dS for S_t = h_t + g_{c(t)} W_{b(t)},
 *   dG_k = sum over t in chunk k of dS_t W_{b(t)}^T,
 *   dW_b = sum over t in bin b of g_{c(t)}^T dS_t   (summed over all rows),
 *   dH_t = dS_t (the residual; the gather adds dG at the boundaries, see
 *          chunk_gather_backward).
 * The Top-K selection itself passes no gradient (notes "Key design 2").
 *
 * dS       fp32 [N, d_l] upstream gradient; offsets NULL (dense) or int64 [rows+1].
 * G        bf16 [total_K, d_g] the chunk vectors of the forward call.
 * idx, idx_offsets, W_bin, nbins, mode: as in chunk_upsample.
 * dG       out fp32 [total_K, d_g]; dW out fp32 [nbins, d_g, d_l] (both
 *          overwritten, zeroed by the call itself).
 * dH       out fp32 [N, d_l] = dS, or NULL to skip the copy.
 * ws       workspace of chunk_upsample_backward_workspace(rows, N, nbins, d_l)
 *          bytes (about 4 d_l + 26 bytes per position).
 * All pointers 16-byte aligned.  Supported: d_g a multiple of 128, d_l a
 * multiple of 64, both up to 4096.  dG and dW are sums of fp32 partial
 * results added with atomics: repeated calls agree to rounding, not bitwise.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA; device flags BOUNDS,
 * TIMEOUT.
 * ------------------------------------------------------------------------- */
DBC_API size_t chunk_upsample_backward_workspace(int64_t rows, int64_t N, int nbins, int64_t d_l);
DBC_API dbc_status chunk_upsample_backward(const float *dS, const void *G, int64_t d_g,
                                           const int64_t *offsets, int64_t T, int64_t N, int64_t d_l,
                                           const int64_t *idx, const int64_t *idx_offsets, int64_t rows,
                                           int64_t total_K, const void *W_bin, int nbins, int mode,
                                           float *dG, float *dW, float *dH, void *ws, size_t ws_bytes,
                                           int32_t *dev_status, dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * chunk_gather_backward -- adjoint of chunk_gather's copy.
 *
 * ByteFlow (summary stage 2): z_k = h_{s_k}, so dL/dh_{s_k} receives dL/dz_k
 * and every other position nothing:
 *   dH[row start + s_k] = dZ_k          (accumulate == 0), or
 *   dH[row start + s_k] += dZ_k         (accumulate != 0, e.g. onto the
 *                                        residual dH of chunk_upsample_backward).
 * Rows of dH that are no boundary are left untouched.
 *
 * dZ       fp32 [total_K, d]; dH in/out fp32 [N, d]; idx, idx_offsets,
 *          offsets as in chunk_gather.  d a multiple of 4; 16-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA; device flag BOUNDS (a boundary
 * outside its row is skipped).
 * ------------------------------------------------------------------------- */
DBC_API dbc_status chunk_gather_backward(const float *dZ, int64_t d, const int64_t *offsets, int64_t T,
                                         const int64_t *idx, const int64_t *idx_offsets, int64_t rows,
                                         int64_t total_K, float *dH, int accumulate, int32_t *dev_status,
                                         dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * chunk_upsample_noalloc -- chunk_upsample for callers that cannot allocate.
 *
 * No passage of the pages corresponds to this entry point; it is a deployment
 * convenience.  Some callers cannot provide device scratch: a host thread
 * inside an inference server whose device memory is entirely owned by the
 * server's own pool, or a plugin/extension point that receives only its input
 * and output buffers and must not call cudaMalloc (which can synchronise the
 * device and fails once the memory budget is taken).  This variant computes
 * exactly what chunk_upsample computes, with the same arguments minus the
 * workspace, and calls no allocating routine (no cudaMalloc/cudaFree, no
 * allocating library call).
 *
 * Its scratch is a built-in static device array of 10 MiB that every GPU
 * loading libdbc.so keeps until the process exits.  Limit: N <= 1048576
 * positions per call; larger N returns DBC_ERR_WORKSPACE before any launch
 * (use chunk_upsample with a caller workspace instead).
 * The first call made with a given device current looks up the array's device
 * address (cudaGetSymbolAddress) and caches it; make that first call before
 * any stream capture.  The cached address belongs to the device's context:
 * after cudaDeviceReset (or any other teardown of that context) it is stale,
 * so do not call this entry point on that device again in the same process.
 * All calls share the one array, which keeps the last
 * call's contents (the call clears what must start at zero): calls that can
 * overlap on the GPU -- concurrent streams or host threads on one device --
 * race on it and must be serialised by the caller.
 * Errors: as chunk_upsample, with DBC_ERR_WORKSPACE for N above the limit.
 * ------------------------------------------------------------------------- */
DBC_API dbc_status chunk_upsample_noalloc(const void *G, int64_t d_g, const void *H, int dtype,
                                          const int64_t *offsets, int64_t T, int64_t N, int64_t d_l,
                                          const int64_t *idx, const int64_t *idx_offsets, int64_t rows,
                                          const void *W_bin, int nbins, int mode, float *S,
                                          int32_t *dev_status, dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * canon_conv1d -- the Canon layer of the local encoder: a causal depthwise
 * convolution with kernel 4 over each row.
 *
 * ByteFlow (notes "Key design 1": every local-encoder layer adds a Canon
 * layer, a causal 1-D convolution of kernel 4; summary "Method steps", stage
 * 1: SWA + Canon(causal_conv1d, k = 4) + SwiGLU, whose output h feeds the
 * chunker).  Reading used (per channel f, positions before a row's start = 0):
 *   out_t[f] = bf16( bias[f] (+ h_t[f] when residual) + sum_{j=0..3} w[f*4+j] h_{t-j}[f] )
 * accumulated in fp32 in that order (bias, residual, taps 0..3), one
 * round-to-nearest-even to bf16.
 *
 * H        bf16 [N, d]; offsets NULL (dense rows of length T) or int64 [rows+1].
 * w        bf16 [d, 4] taps (w[f*4 + j] multiplies h_{t-j}); bias bf16 [d] or NULL.
 * out      bf16 [N, d], must not overlap H.  H and out 16-byte aligned.
 * Supported: d a multiple of 8 up to 4096.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA; device flag BOUNDS (malformed offsets).
 * ------------------------------------------------------------------------- */
DBC_API dbc_status canon_conv1d(const void *H, const int64_t *offsets, int64_t rows, int64_t T, int64_t N,
                                int64_t d, const void *w, const void *bias, int residual, void *out,
                                int32_t *dev_status, dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * chunk_coding_rate_canon -- canon_conv1d followed by chunk_coding_rate on its
 * output, in one call (the chunker's input is the Canon layer's output).
 *
 * Writes Hc = canon_conv1d(H, ...) (bf16 [N, d], kept for the gather and the
 * upsampling's residual) and dR = the coding rate of Hc.  d in {64, 128, 256,
 * 512}; ws of chunk_coding_rate_workspace(rows, T, N, d) bytes.
 * Errors: as canon_conv1d and chunk_coding_rate.
 * ------------------------------------------------------------------------- */
DBC_API dbc_status chunk_coding_rate_canon(const void *H, const int64_t *offsets, int64_t rows, int64_t T,
                                           int64_t N, int64_t d, const void *w, const void *bias, int residual,
                                           void *Hc, float eps2, float *dR, void *ws, size_t ws_bytes,
                                           int32_t *dev_status, dbc_stream_t stream);

/* -------------------------------------------------------------------------
 * hnet_route -- cosine-similarity boundary router with EMA smoothing.
 *
 * ByteGen report ("H-Net architecture", "Methodology"): boundary probability
 * from the cosine similarity of adjacent byte representations; exponentially
 * weighted smoothing over the chunks.  Reading used (row vectors, per row):
 *   q_t = h_t W_q, k_t = h_t W_k, p_t = 1/2 (1 - cos(q_t, k_{t-1})), p_0 = 1,
 *   b_t = [p_t >= threshold] (cos = 0 when a norm is 0),
 *   chunks: the positions with b_t = 1, in order; per chunk j of a row,
 *   zbar_j = P_j h_{t_j} + (1 - P_j) zbar_{j-1}, P_j = p_{t_j}, zbar_{-1} = 0.
 *
 * H        bf16 [N, d]; Wq, Wk bf16 [d, d] row-major.
 * p        out fp32 [N]; boundary out uint8 [N] (0/1).
 * chunk_idx out int64 [N] capacity: row-relative chunk start positions, rows
 *          stacked; chunk_offsets out int64 [rows+1].
 * z_smooth out fp32 [N, d] capacity (rows stacked like chunk_idx); only
 *          written when do_ema != 0 (may be NULL otherwise).
 * ws       workspace of hnet_route_workspace(rows, N, d) bytes.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA; device flag NONFINITE.
 * ------------------------------------------------------------------------- */
DBC_API size_t hnet_route_workspace(int64_t rows, int64_t N, int64_t d);
DBC_API dbc_status hnet_route(const void *H, const int64_t *offsets, int64_t rows, int64_t T,
                      int64_t N, int64_t d, const void *Wq, const void *Wk,
                      float threshold, int do_ema, float *p, uint8_t *boundary,
                      int64_t *chunk_idx, int64_t *chunk_offsets, float *z_smooth,
                      void *ws, size_t ws_bytes, int32_t *dev_status,
                      dbc_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DBC_H_ */
