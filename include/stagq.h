/*
 * stagq.h -- C ABI of the StagQ multi-precision GEMV library (libstagq.so).
 *
 * The operation (StagQ paper, "StagQ: Constraint-Driven Multi-Precision Weight
 * Quantization for LLMs", arXiv 2610.05977):
 *
 *   y = W_hat^(M) x,   W_hat^(M) = (1 - m) .* (lo_M + s_M u_M) + P          (Eq. 4, 10)
 *
 * u_M is the composite integer of the first M-2 refinement planes on top of
 * the 2-bit base (Eq. 8); (lo_M, s_M) follow in closed form from one 8-bit
 * (lo, s) pair per group (Section 3.1, Eq. 10); m / P is the sparse side
 * record of held-out weights (Eq. 4). The read precision M ("bits") is
 * chosen per call, from 2 up to 2 + n_planes, from ONE stored stream; a
 * p_M read touches only the base and the first M-2 planes (Section 3.3).
 *
 * Conventions for every entry point:
 *  - Shapes are out x in (row = output channel; K = in). Groups are runs of
 *    `group` consecutive weights along K inside one row.
 *  - fp16 values are passed as IEEE binary16 bit patterns (uint16_t).
 *  - Functions return a status code (STAGQ_OK = 0 on success); no C++
 *    exception crosses this boundary. stagq_last_error() gives a detail
 *    message for the calling thread's most recent failure.
 *  - Pointers documented as "host" must be host memory; "device" must be
 *    device memory of the handle's GPU. The library never frees a caller's
 *    pointer.
 */
#ifndef STAGQ_H
#define STAGQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status */
#define STAGQ_OK 0
#define STAGQ_EINVAL 1   /* bad argument: null pointer, bits out of range, n out of range, bad shape */
#define STAGQ_EFORMAT 2  /* malformed stream: row_ptr not monotone, col >= in, bad file header */
#define STAGQ_ENOMEM 3   /* host or device allocation failed */
#define STAGQ_ECUDA 4    /* a CUDA runtime call failed (detail in stagq_last_error) */
#define STAGQ_EIO 5      /* file could not be read or written */
#define STAGQ_ENODEV 6   /* no usable sm_100 device */
#define STAGQ_ETIMEOUT 7 /* a GEMV kernel gave up waiting for its own copies (reported by stagq_check) */

/* Limits of this implementation. */
#define STAGQ_MAX_PLANES 4      /* stream depth N = 2 + n_planes <= 6 (the paper evaluates N = 6) */
#define STAGQ_MAX_BATCH 4       /* columns of x per call in stagq_gemv_n */
#define STAGQ_MAX_STACK 4       /* member matrices of one stacked handle (stagq_load_stack) */
#define STAGQ_MAX_IN 32768      /* K; side-record columns are stored as uint16 */
#define STAGQ_IN_MULTIPLE 128   /* K must be a multiple of this (16-byte plane rows) */
/* The group size of a loadable stream is a power of two, at least this, dividing
 * K. Groups of 16 and 32 are the paper's encoder settings (Table 6), and its
 * kernel evaluation runs at 32 (Section 4.3, Table 5), where the 8-bit pair
 * costs 0.25 bpw; the kernels then apply G = 64 / group affines per
 * 64-weight chunk. */
#define STAGQ_MIN_GROUP 16

/* Pair search mode of the encoder (Section 3.1). */
#define STAGQ_PAIR_SEARCH 0     /* argmin of Eq. (5) over all 256 codebook pairs */
#define STAGQ_PAIR_FAST 1       /* nearest codebook entry per coordinate (labelled shortcut) */
/* OR'ed into the pair mode: codebooks by Appendix E's rules -- of the nine
 * combinations of uniform, Lloyd and anchored-Lloyd placement for the two
 * codebooks, the one with the smallest summed first term of Eq. (5); uniform
 * placement instead if, under it, the deepest precision's error exceeds a
 * tenth of the two-bit error. Without it both codebooks are uniform. */
#define STAGQ_CODEBOOK_RULES 0x100

/* Flags of stagq_gemv_ex. */
#define STAGQ_Y_F32 1u          /* y is fp32 instead of fp16 */
/* Kernel choice (default: by shape and vector count, see stagq_gemv_ex). */
#define STAGQ_KERNEL_GENERAL 2u /* the kernel of any vector count (one or two CTAs per SM) */
#define STAGQ_KERNEL_SINGLE 4u  /* the single-vector kernel (one CTA per SM, with the SM to itself) */

typedef struct stagq_matrix* stagq_handle;   /* opaque; owned by the library */

/*
 * Logical fields of one encoded matrix (Sections 3.3-3.6): one byte per
 * digit, no physical layout. Filled by stagq_encode, consumed by stagq_pack.
 * All arrays are host memory owned by the caller.
 *   q         [out*in]            base digit 0..3, row-major
 *   planes    [n_planes*out*in]   b_k in {0,1}; plane k (k = 3..2+n_planes) at offset (k-3)*out*in
 *   pair_idx  [out*(in/group)]    8-bit pair: high nibble = log2(s) codebook index, low = lo/s index
 *   row_ptr   [out+1]             side record (CSR): entries of row r are [row_ptr[r], row_ptr[r+1])
 *   col       [nnz]               column of each held-out weight, increasing inside a row;
 *                                 bit 15 (STAGQ_SIDE_POST) marks a post-grid entry
 *   val       [nnz]               fp16: the recorded value (pre-grid entry, P = val) or the
 *                                 residual r against the two-bit reconstruction (post-grid
 *                                 entry, P = lo + s q + r; Section 3 below Eq. 4)
 * Pre-grid positions carry zero digits (q = 0, all b_k = 0); post-grid
 * positions keep their base digit q and carry zero planes.
 */
#define STAGQ_SIDE_POST 0x8000u
typedef struct {
    int32_t out, in, group, n_planes;
    int64_t nnz;
    uint16_t codebook_log2s[16];
    uint16_t codebook_lo_over_s[16];
    uint8_t* q;
    uint8_t* planes;
    uint8_t* pair_idx;
    int32_t* row_ptr;
    uint16_t* col;
    uint16_t* val;
} stagq_fields;

/*
 * Packed, plane-major stream (Section 3.3: base first, then the planes in
 * order of k, so a shallower read skips the deeper planes). Host memory,
 * owned by the caller.
 *   planes: stagq_stream_plane_bytes(out, in, n_planes) bytes =
 *           [base: out*in/4 B][plane 3: out*in/8 B]...[plane 2+n_planes: out*in/8 B]
 *           Each plane is row-major; inside a row the weights are stored in
 *           64-weight lane chunks whose bit order is the library's own.
 *   pair_idx, row_ptr, col, val: as in stagq_fields.
 */
typedef struct {
    int32_t out, in, group, n_planes;
    int64_t nnz;
    uint16_t codebook_log2s[16];
    uint16_t codebook_lo_over_s[16];
    const uint8_t* planes;
    const uint8_t* pair_idx;
    const int32_t* row_ptr;
    const uint16_t* col;
    const uint16_t* val;
} stagq_host_stream;

typedef struct {
    int32_t out, in, group, n_planes;
    int64_t nnz;
    int32_t device;
    int64_t device_bytes;     /* bytes the handle holds on the GPU */
} stagq_info_t;

/* ------------------------------------------------------------- encoding */

/* Number of side-record entries for a density: round(density*out*in), half up. */
int64_t stagq_side_record_count(int32_t out, int32_t in, double density);

/*
 * Side-record capacity of stagq_encode_guarded: one pre-grid entry per group
 * and one post-grid entry per row at most, out*(in/group) + out.
 */
int64_t stagq_guard_capacity(int32_t out, int32_t in, int32_t group);

/*
 * The encoder with the paper's guards in place of the density record:
 * pre-grid ratio criterion (Section 3.5: a group's largest-|w| entry is held
 * out when it exceeds ratio_T times the second largest; T = 4 on
 * Llama-3.1-8B, Table 6) and, if post_guard != 0, the post-grid guard of a
 * ratio-criterion matrix (Appendix E: per row, the position with the largest
 * two-bit error (w - (lo + s q))^2 under the fitted grid, recorded as an
 * fp16 residual with STAGQ_SIDE_POST in its column). The rest is
 * stagq_encode's steps 2-7.
 *   f->nnz   in: capacity of f->col / f->val, at least stagq_guard_capacity();
 *            out: the entries written.
 * Errors: as stagq_encode; STAGQ_EINVAL if ratio_T < 1 or the capacity is short.
 */
int stagq_encode_guarded(const uint16_t* w, double ratio_T, int32_t post_guard, int32_t pair_mode,
                         int32_t n_threads, stagq_fields* f);

/*
 * Encoder of Sections 3.1-3.6 / Appendices B, E for a synthetic fp16 matrix
 * (host, multithreaded): global top-|w| side record with `density`, held-out
 * entries clipped inward for the fit, initial pair (Appendix B), fp16
 * codebooks (Appendix E: uniform placement, or Appendix E's rules with
 * STAGQ_CODEBOOK_RULES OR'ed into `pair_mode`), pair per group by `pair_mode`
 * (STAGQ_PAIR_SEARCH / STAGQ_PAIR_FAST), nearest-rounding base, sign planes
 * (Eq. 7), zero digits at held-out positions.
 *   w        host [out*in] fp16 bits, row-major
 *   f        caller sets out, in, group, n_planes and points every array at a
 *            buffer of the documented size, with nnz = stagq_side_record_count(...);
 *            the encoder fills codebooks and arrays.
 *   n_threads  0 = all hardware threads.
 * Errors: STAGQ_EINVAL (null, group does not divide in, n_planes > STAGQ_MAX_PLANES,
 *         nnz mismatch, in > STAGQ_MAX_IN, unknown pair-mode bits), STAGQ_ENOMEM.
 */
int stagq_encode(const uint16_t* w, double density, int32_t pair_mode, int32_t n_threads,
                 stagq_fields* f);

/* Size in bytes of the packed plane region: out*in/4 + n_planes*out*in/8. */
int64_t stagq_stream_plane_bytes(int32_t out, int32_t in, int32_t n_planes);

/*
 * Packer (host): lays the logical digits of `f` out plane-major into
 * `planes_out` (stagq_stream_plane_bytes bytes, caller-owned).
 * Errors: STAGQ_EINVAL (null, in not a multiple of STAGQ_IN_MULTIPLE, digit out of range).
 */
int stagq_pack(const stagq_fields* f, uint8_t* planes_out);

/*
 * Host re-read of a packed stream: u_M (Eq. 8) per weight into u_out
 * (host [out*in], row-major), using the same bit manipulations as the GPU
 * kernels. For checking a stream on a machine without a GPU; no GEMV runs here.
 */
int stagq_unpack_levels_host(const stagq_host_stream* s, int bits, uint8_t* u_out);

/* Serialise a stream to a file (one checkpoint serving every precision,
 * Section 1) and read it back straight onto a GPU. */
int stagq_save(const stagq_host_stream* s, const char* path);
int stagq_load_file(const char* path, int device, stagq_handle* out);

/* ------------------------------------------------------------ the GEMV */

/*
 * Copy a stream to GPU `device` and build the per-precision (lo_M, s_M)
 * tables (Eq. 10, computed in fp64 on the host, stored fp32).
 * The caller keeps ownership of every host array; the handle owns its device
 * copies until stagq_free.
 * Errors: STAGQ_EINVAL, STAGQ_EFORMAT (row_ptr not monotone or not ending at
 * nnz, col >= in), STAGQ_ENOMEM, STAGQ_ENODEV, STAGQ_ECUDA.
 */
int stagq_load(const stagq_host_stream* s, int device, stagq_handle* out);

/*
 * One handle for up to STAGQ_MAX_STACK matrices that are applied to the same
 * x (a transformer layer's q/k/v projections, or gate/up): member j's rows
 * follow member j-1's, so the handle is one (sum of outs) x in matrix and
 * every GEMV entry point serves all members in one launch, with y the
 * members' outputs one after the other. Each member keeps its own
 * codebooks (the paper fits them per matrix, Section 3.1), pair bytes and
 * side record; the members must share in, group and n_planes. The result of
 * member j's rows equals what a handle of member j alone computes (same
 * arithmetic per row). stagq_bytes counts x once.
 *   members   host array of `count` streams (1 <= count <= STAGQ_MAX_STACK);
 *             the caller keeps ownership of everything they point to.
 * Errors: STAGQ_EINVAL (count, null, members that differ in in / group /
 * n_planes), the errors of stagq_load.
 */
int stagq_load_stack(const stagq_host_stream* const* members, int count, int device, stagq_handle* out);

/*
 * y = W_hat^(bits) x for one vector (n = 1), asynchronously on `cuda_stream`
 * (a cudaStream_t; NULL = the legacy default stream).
 *   bits   2 .. 2 + n_planes
 *   x      device [in]  fp16
 *   y      device [out] fp16 (fp32 accumulation, rounded to nearest even)
 * Calls on one handle may run concurrently: the GEMV uses no scratch memory
 * (each CTA stages its rows in its own shared memory).
 * Errors: STAGQ_EINVAL (null handle/pointer, bits out of range), STAGQ_ECUDA (launch failure).
 */
int stagq_gemv(stagq_handle h, int bits, const void* x, void* y, void* cuda_stream);

/* n columns (1 <= n <= STAGQ_MAX_BATCH): x device [n*in], y device [n*out], row-major. */
int stagq_gemv_n(stagq_handle h, int bits, const void* x, int n, void* y, void* cuda_stream);

/*
 * As stagq_gemv_n; flags STAGQ_Y_F32 makes y fp32. The library has two
 * kernels with the same integer dot products (results agree to fp32
 * rounding, each is deterministic). By default the single-vector kernel
 * serves every call it can plan, where it measured faster:
 *   - n = 1 with K <= 30720;
 *   - n = 2..4 with K <= 15360 and groups of 64 or more.
 * The general kernel serves the rest.
 * STAGQ_KERNEL_GENERAL / STAGQ_KERNEL_SINGLE force one of them, for tests and
 * measurements. Forcing the single-vector kernel on a shape and n it cannot
 * plan returns STAGQ_EINVAL.
 */
int stagq_gemv_ex(stagq_handle h, int bits, const void* x, int n, void* y, uint32_t flags,
                  void* cuda_stream);

/*
 * As stagq_gemv_ex with the run-time inverse activation scale (Appendix E:
 * the quantiser saw W diag(a), so the decoder multiplies channel c of x by
 * 1/a_c): y_j = W_hat^(bits) (x_j .* in_scale) for each of the n vectors.
 *   in_scale  device [in] fp32 (the values 1/a_c), 16-byte aligned.
 * The product x_c in_scale_c is rounded to fp32, then converted like x
 * (separate kernel instances: calls without a scale keep their code).
 * Errors: as stagq_gemv_ex; STAGQ_EINVAL for a null or misaligned in_scale.
 */
int stagq_gemv_scaled(stagq_handle h, int bits, const void* x, int n, const float* in_scale, void* y,
                      uint32_t flags, void* cuda_stream);

/*
 * End-to-end call with HOST buffers: copies x (host [n*in] fp16) to the
 * device, runs the GEMV and copies y (host [n*out] fp16) back, all on
 * `cuda_stream`, and returns after the copy of y has completed. Uses a
 * device staging buffer owned by the handle, so calls on one handle must
 * not overlap.
 */
int stagq_gemv_host(stagq_handle h, int bits, const void* x_host, int n, void* y_host,
                    void* cuda_stream);

/*
 * Several GEMVs with HOST buffers and one synchronization: for i in
 * [0, count), copies x_hosts[i] (host [ns[i]*in_i] fp16) to the device, then
 * runs y_i = W_hat_i^(bits[i]) x_i with handle hs[i] (ns[i] = 1..4 vectors),
 * then copies y_i back to y_hosts[i] (host [ns[i]*out_i] fp16). Every copy
 * and launch goes on `cuda_stream` in that order: all x copies, all GEMVs (so
 * consecutive launches overlap as in a device-side chain), all y copies. The
 * call returns after the last copy of y has completed.
 *   - Handles may repeat, and every handle must live on the same device.
 *   - count is 1..STAGQ_MAX_MANY.
 *   - Pinned host memory makes the copies asynchronous; pageable memory also
 *     works.
 *   - The device staging buffer is owned by the library, one per device. It
 *     is allocated on first use and grown as needed. Calls on one device must
 *     not overlap.
 * Errors: STAGQ_EINVAL for a bad count, a null array or pointer, an n outside
 * 1..STAGQ_MAX_BATCH, or handles on different devices; as stagq_gemv_ex for
 * the GEMVs; STAGQ_ENOMEM if staging cannot be allocated. On an error no y_i
 * is guaranteed to be written.
 */
#define STAGQ_MAX_MANY 1024
int stagq_gemv_host_many(int count, const stagq_handle* hs, const int* bits, const void* const* x_hosts,
                         const int* ns, void* const* y_hosts, void* cuda_stream);

/*
 * As stagq_gemv_host, but allocates nothing: x and y are staged through a
 * statically reserved device array of STAGQ_NOALLOC_STAGE_BYTES (x in its
 * first 256 KiB, y in the rest), where stagq_gemv_host would cudaMalloc a
 * staging buffer on first use. For callers that must not allocate device
 * memory while they run: under a fixed device-memory budget owned by another
 * allocator, or in a phase where new allocations are forbidden. The paper has
 * no counterpart; this is a property of this library's host interface.
 *   - The array exists on every GPU that loads the library and is held until
 *     the process exits.
 *   - Every call looks up the array's device address with the handle's
 *     device current (cudaGetSymbolAddress; nothing is cached, so a device
 *     reset in between is harmless). The first call on a device may also
 *     load the library's device code there; make that first call before any
 *     stream capture.
 *   - All calls share the one array, which keeps the last call's contents
 *     (nothing of it is read before being written). Calls that overlap on the
 *     GPU race: issue them one at a time. The call returns after the copy of y
 *     has completed.
 * Errors: as stagq_gemv_host; STAGQ_EINVAL when n*out*2 bytes of y exceed
 * STAGQ_NOALLOC_STAGE_BYTES - 256 KiB (x always fits: n*in*2 <= 256 KiB).
 */
#define STAGQ_NOALLOC_STAGE_BYTES (2u << 20)
int stagq_gemv_host_noalloc(stagq_handle h, int bits, const void* x_host, int n, void* y_host,
                            void* cuda_stream);

/* Test hook: u_M per weight (device [out*in] uint8, row-major), decoded on the GPU. */
int stagq_decode_levels(stagq_handle h, int bits, uint8_t* u_dev, void* cuda_stream);

/*
 * Algorithmic bytes of one call (the roofline numerator):
 *   out*in*bits/8 (base + bits-2 planes) + out*in/group (pairs)
 *   + 4*nnz + 4*(out+1) (side record) + 2*n*in (x) + 2*n*out (y).
 * Returns -1 for a bad handle or bits.
 */
int64_t stagq_bytes(stagq_handle h, int bits, int n);

/*
 * Synchronise the handle's device and report any CUDA error raised by work
 * queued on it (the GEMV entry points are asynchronous and only report launch
 * errors), then whether a GEMV on this handle gave up waiting for its own
 * copies since the last check (every wait inside the kernel is bounded to
 * 2 s; on expiry the kernel sets the handle's status word, lets its copies in
 * flight land and returns, leaving y undefined). Clears the status word.
 * Returns STAGQ_OK, STAGQ_ETIMEOUT or STAGQ_ECUDA.
 */
int stagq_check(stagq_handle h);

int stagq_info(stagq_handle h, stagq_info_t* info);

/* ------------------------------------------------------------ test hooks */

/*
 * Test hook for the bounded waits: while stall_ns != 0, every GEMV launched
 * on the handle (its arguments are taken at launch, so a captured CUDA graph
 * keeps the value of its capture) first waits at most stall_ns on a barrier
 * that nothing completes. The wait runs out, the kernel takes its give-up
 * path -- it lets its own copies in flight land, sets the handle's status
 * word and returns without writing y -- and the next stagq_check returns
 * STAGQ_ETIMEOUT. No GPU fault is involved. 0 turns the hook off.
 */
int stagq_debug_stall(stagq_handle h, uint32_t stall_ns);

/*
 * Where the handle's side record lives on the device: the loader re-lays the
 * CSR record (Eq. 4) per CTA for each kernel's grid.
 *   General kernel (grid CTAs, stride bytes each): CTA b owns rows
 *   [b out / grid, (b + 1) out / grid); its rows fall in row_groups classes
 *   (local row mod row_groups); int32 offsets [row_groups][k_slices]
 *   [class_rows + 1] give where row m of a class starts within the run of
 *   its (class, K slice) -- a K slice is 2048 columns -- and the run's end;
 *   entries (uint32: column with the post-grid flag in bit 15 | fp16 value
 *   << 16) start at ent_off.
 *   Single-vector kernel (grid1 CTAs, stride1 bytes each, same row split):
 *   int32 offsets [rows + 1] per local row, entries at ent_off1 in (row,
 *   column) order, same word.
 */
typedef struct {
    int32_t grid, stride, ent_off, row_groups, k_slices, class_rows;
    int32_t grid1, stride1, ent_off1;
} stagq_side_layout_t;

/*
 * Test hook: fills *layout and copies the two device cuts of the side record
 * to host memory (grid * stride and grid1 * stride1 bytes; a null buffer is
 * skipped), so that a test can check them entry by entry against the CSR.
 * Errors: STAGQ_EINVAL (null handle or layout, a buffer below its size),
 * STAGQ_ECUDA.
 */
int stagq_debug_side_record(stagq_handle h, stagq_side_layout_t* layout, void* cut_host, int64_t cut_bytes,
                            void* cut1_host, int64_t cut1_bytes);

/* Release the handle's device memory. Null-safe. */
void stagq_free(stagq_handle h);

const char* stagq_strerror(int status);
const char* stagq_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* STAGQ_H */
