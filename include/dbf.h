/*
 * dbf.h — C ABI of libdbf, a single-GPU (B200, sm_100a) implementation of the
 * Double Binary Factorization (DBF) linear-layer forward pass.
 *
 * The method ("Addition is almost all you need: Compressing large language
 * models with double binary factorization"; gist.science technical summary,
 * section 2.1; sciencestack.ai Figure 1) replaces a dense weight W (n x m_in) by
 *
 *     W ~= (a (.) A (.) mid^T)(B (.) b^T)
 *
 * with A in {+-1}^(n x k), B in {+-1}^(k x m_in) and fp16 scale vectors a (n),
 * mid (k), b (m_in).  ("mid" is the middle vector the pages call m; it is named
 * m in the argument lists below.)  The forward of an input batch X is evaluated
 * in the order the pages give, so that both sign products are additions and
 * sign flips:
 *
 *     Y = X W^T ~= ((((X (.) b^T) B^T) (.) mid^T) A^T) (.) a^T
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All data pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates, frees or keeps memory; apart from cached device properties
 *    it keeps no state between calls (dbf_forward_noalloc aside, see there).
 *  - fp16 buffers are IEEE binary16 bit patterns (uint16_t), e.g. __half or a
 *    torch.float16 tensor.
 *  - Matrices are row-major and dense (no padding between rows) unless said.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  A call returns after enqueueing.
 *  - Synchronous argument checks run first; a call that returns anything but
 *    DBF_OK has enqueued nothing.  DBF_ERR_CUDA reports a failed launch; faults
 *    that happen later on the device surface through the stream (and, for
 *    dbf_forward, the workspace status word, see dbf_workspace_status).
 *  - No C++ exception crosses this interface.
 *
 * Packed sign layout (the pages only say the factors are binary sign
 * matrices; this bit layout is the library's own choice):
 *  - A rows x cols sign matrix is stored row after row.  Each row occupies
 *    dbf_packed_words_per_row(cols) = ceil(cols/256)*8 little-endian 32-bit
 *    words: one block of 8 words per 256 columns, so every row starts on a
 *    32-byte boundary.
 *  - Inside a block, column e (0..255) belongs to group g = e/16 and pair
 *    p = (e%16)/2 of that group.  It is held in word p of the block at bit
 *    g + 16*(e%2).  Word p therefore carries, at bits (g, g+16), the column
 *    pair (16g + 2p, 16g + 2p + 1) of every group g: one shift and one mask
 *    turn it into an fp16 pair of signs, and the 16 columns of a group come
 *    from the same bit pair of the block's 8 words.
 *  - A set bit means -1, a clear bit +1.  Bits past the last column are 0.
 *  - packedA holds A (n rows over k columns); packedB holds B (k rows over
 *    m_in columns): both are packed along the reduction dimension of their
 *    product.
 */
#ifndef DBF_H_
#define DBF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* the type a cudaStream_t points to */

#if defined(__GNUC__)
#define DBF_API __attribute__((visibility("default")))
#else
#define DBF_API
#endif

typedef enum dbf_status {
  DBF_OK = 0,
  DBF_ERR_INVALID_ARG = 1,       /* null pointer, negative size, unknown enum, bad flag */
  DBF_ERR_UNSUPPORTED_SHAPE = 2, /* outside the shape contract of the call */
  DBF_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
  DBF_ERR_WORKSPACE = 4,         /* workspace null, misaligned or smaller than required */
  DBF_ERR_CUDA = 5,              /* a CUDA runtime call or kernel launch failed */
  DBF_ERR_TIMEOUT = 6,           /* a bounded device-side wait gave up (status word) */
  DBF_ERR_DEVICE = 7             /* the current device is not an sm_100 (B200-class) GPU */
} dbf_status;

typedef enum dbf_dtype { DBF_I8 = 0, DBF_F16 = 1, DBF_F32 = 2 } dbf_dtype;

/* dbf_forward flags (bitwise OR; 0 is the safe default). */
enum {
  /* The packed signs and the three scale vectors are not written by any work
   * that may still be running on `stream` when this call is enqueued (true for
   * inference weights loaded ahead of time).  The kernels may then start
   * streaming weights before the previous kernel on the stream has finished
   * (programmatic dependent launch).  x is always read only after it. */
  DBF_FWD_WEIGHTS_STATIC = 1u << 0,
  /* Force the batch <= 16 sign-GEMV path (batches above 16 run in chunks of 16). */
  DBF_FWD_FORCE_DECODE = 1u << 1,
  /* Force the tensor-core (tcgen05) path at any batch size. */
  DBF_FWD_FORCE_PREFILL = 1u << 2,
  /* Two-launch decode path: form the fp16 sign operands by shift+mask with
   * one accumulator set instead of the default bit-position classes (implies
   * DBF_FWD_DECODE_TWO_STAGE). */
  DBF_FWD_DECODE_SHIFT_EXPAND = 1u << 3,
  /* Decode path: run the two products as two PDL-chained launches (fp16
   * tensor-core sign-GEMV) instead of the single-launch kernel. */
  DBF_FWD_DECODE_TWO_STAGE = 1u << 4,
  /* Decode path: run the whole layer as one launch (int8 tensor-core sign
   * products in block fixed point, the middle vector exchanged inside
   * thread-block clusters) wherever the shape fits it, instead of the
   * library's choice between the two decode kernels. */
  DBF_FWD_DECODE_SINGLE = 1u << 5,
  /* Decode path, one token: form the products by table lookup instead of the
   * fp16 warp-MMA sign-GEMV: per nibble of packed signs a table of the 16
   * signed sums of the four activations it selects, built in fp32 from
   * u = x (.) b (so u is not rounded to fp16; V still is).  Slower than the
   * default on most layer shapes, faster on layers of about 1000 rows; no
   * effect above one token.  Not with DBF_FWD_DECODE_SHIFT_EXPAND or
   * DBF_FWD_DECODE_SINGLE. */
  DBF_FWD_DECODE_TABLE = 1u << 6,
  /* TEST ONLY.  Makes one bounded wait of the single-launch decode kernel run
   * out (rank 0 of each cluster waits for 16 bytes that are never sent), so
   * that failure reporting can be tested without a fault: the call still
   * returns DBF_OK, the kernel ends after the wait budget (about 0.2-0.4 s)
   * with y unwritten, and the workspace status word reads DBF_ERR_TIMEOUT.
   * The workspace must then be zero-filled again before its next use. */
  DBF_FWD_TEST_LOSE_ARRIVAL = 1u << 30
};

/* Words (uint32) in one packed row of `cols` signs: ceil(cols/256)*8.
 * Returns 0 for cols <= 0. */
DBF_API int64_t dbf_packed_words_per_row(int64_t cols);

/* Words (uint32) of a packed rows x cols sign matrix: rows*ceil(cols/256)*8.
 * Returns 0 for rows <= 0 or cols <= 0. */
DBF_API int64_t dbf_packed_words(int64_t rows, int64_t cols);

/*
 * Pack a sign matrix into the layout above (the pages' storage format: A and
 * B hold only +-1 entries, sciencestack.ai Figure 1; gist.science section 2.1).
 *   src     rows x cols, row-major, element type src_t (DBF_I8, DBF_F16 or
 *           DBF_F32).  An element packs to -1 (set bit) iff it compares < 0;
 *           0, -0.0 and NaN pack to +1.
 *   packed  dbf_packed_words(rows, cols) words, written in full (padding bits
 *           are cleared).  Must be 16-byte aligned and must not overlap src.
 * Shape: rows >= 1, cols >= 1.  Any cols is accepted here; dbf_forward itself
 * needs k and m_in to be multiples of 64.
 */
DBF_API dbf_status dbf_pack_signs(const void* src, dbf_dtype src_t, int64_t rows, int64_t cols,
                          uint32_t* packed, struct CUstream_st* stream);

/*
 * Workspace bytes that let dbf_forward run every schedule for these sizes
 * (0 if a size is < 1).  Layout: a 256-byte status block (an int32 status
 * word at offset 0); the middle activations V = fp16(mid (.) (B (x (.) b))) as
 * batch x k fp16, padded to 256 bytes; then an optional area:
 *   batch <= 16: the single-launch decode's tagged partials, 8 x batch x n
 *                64-bit words (used with DBF_FWD_DECODE_SINGLE);
 *   batch > 128: the tensor-core path's stream-K area, 1 KiB of flags and 160
 *                partial tiles of 128 x 256 fp32 (20,972,544 bytes), used for
 *                the GEMMs whose tiles would leave a partial last wave.
 * dbf_forward accepts any workspace of at least 256 + round_up(batch*k*2, 256)
 * bytes and runs a schedule that needs no optional area when it is smaller
 * than this size.
 * The workspace must be zero-filled before its first use.  After a call that
 * leaves the status word at 0 it can be reused as it is (the library returns
 * every flag it raises to zero; the status word changes only when a
 * device-side wait gives up, after which the workspace must be zero-filled
 * again).  Calls that may run concurrently need distinct workspaces.
 */
DBF_API size_t dbf_forward_workspace_bytes(int64_t n, int64_t k, int64_t m_in, int64_t batch);

/*
 * y = ((((x (.) b^T) B^T) (.) m^T) A^T) (.) a^T    (section 2.1, computation
 * process; both sign products are evaluated without materialising W).
 *
 *   x          batch x m_in fp16, row-major.
 *   packedA    A in the packed layout, n rows over k.
 *   packedB    B in the packed layout, k rows over m_in.
 *   a, m, b    fp16 vectors of n, k and m_in entries (m is the pages' middle
 *              vector, "mid" above).
 *   y          batch x n, row-major, y_t = DBF_F16 (round to nearest even,
 *              overflow to +-inf) or DBF_F32.
 *   workspace  ws_bytes >= 256 + round_up(batch*k*2, 256); the size
 *              dbf_forward_workspace_bytes(n, k, m_in, batch) enables every
 *              schedule.  Zero-filled before its first use (see above).
 *   flags      DBF_FWD_* bits.
 * Arithmetic: both sign products accumulate in fp32.  The middle vector V is
 * rounded to fp16 once (V = fp16(mid (.) t)); the decode path also rounds
 * x (.) b to fp16 before the first product, the tensor-core path folds b into
 * the sign operand exactly.  With a = m = b = 1, integer x and |t| <= 2048,
 * every step is exact and fp32 output equals the integer result.
 * Paths: batch <= 16 runs two PDL-chained sign-GEMV kernels (mma.sync);
 * larger batches run the two products as tcgen05 tensor-core GEMMs, one
 * launch each, or two when a GEMM's last wave of tiles would leave most SMs
 * idle (its last rows then run as a split-K launch of their own).  Past 128
 * tokens a GEMM whose tiles do not fill whole waves may instead run stream-K
 * (one contiguous range of (tile, K block) units per SM; a tile split between
 * CTAs is completed by the CTA holding its first K blocks, which adds the
 * others' fp32 partial tiles in a fixed order): results then differ from the
 * one-launch schedule only in the grouping of fp32 additions, and are
 * identical in integer mode.  Stream-K waits on other CTAs of its own grid
 * (bounded, DBF_ERR_TIMEOUT): its CTAs, one per SM, must all become resident
 * within the wait budget, so it should not share the GPU with kernels that
 * hold SMs for longer.
 * Shape contract: n >= 1, batch >= 1, k and m_in multiples of 64 in
 * [64, 1 << 20], n and batch <= 1 << 24.  All pointers 16-byte aligned;
 * outputs must not overlap inputs.
 */
DBF_API dbf_status dbf_forward(const uint16_t* x, const uint32_t* packedA, const uint32_t* packedB,
                       const uint16_t* a, const uint16_t* m, const uint16_t* b, int64_t n, int64_t k,
                       int64_t m_in, int64_t batch, void* y, dbf_dtype y_t, void* workspace,
                       size_t ws_bytes, uint32_t flags, struct CUstream_st* stream);

/*
 * Dense reconstruction W = (a (.) A (.) m^T)(B (.) b^T), n x m_in row-major
 * (section 2.1, factorisation equation):
 *     W[i][j] = a_i * b_j * sum_l A[i][l] m_l B[l][j]   (fp32 accumulation)
 * W_t is DBF_F16 (round to nearest even) or DBF_F32.  Not a hot path: it
 * exists to check a factorisation against the dense weight it stands for.
 * Shape contract as dbf_forward (k, m_in multiples of 64); pointers 16-byte
 * aligned.
 */
DBF_API dbf_status dbf_reconstruct_dense(const uint32_t* packedA, const uint32_t* packedB, const uint16_t* a,
                                 const uint16_t* m, const uint16_t* b, int64_t n, int64_t k, int64_t m_in,
                                 void* W, dbf_dtype W_t, struct CUstream_st* stream);

/*
 * Copy the workspace status word to *device_status (synchronises `stream`).
 * 0 means no device-side wait has given up since the workspace was zeroed;
 * otherwise it holds the dbf_status of the first failure (DBF_ERR_TIMEOUT).
 */
DBF_API dbf_status dbf_workspace_status(const void* workspace, struct CUstream_st* stream, int32_t* device_status);

/*
 * dbf_forward for callers that cannot allocate device memory.  (The pages have
 * no counterpart: this concerns who provides the scratch buffer, not the
 * method.)  Some callers have no allocator to hand: a plugin inside a host
 * application that owns all device memory and offers its extensions none, or
 * a latency-critical thread that must not call cudaMalloc (which can block
 * and synchronise the device).  This call takes the same arguments as
 * dbf_forward minus the workspace and uses instead a 2 MiB buffer that lives
 * in the library (a static __device__ array, held by every GPU that loads the
 * library until the process exits).  It allocates and frees nothing.
 *   Limit: the smallest workspace dbf_forward accepts, 256 + batch*k*2 bytes
 *   (rounded up to 256), must fit in 2 MiB (e.g. batch 16 with k up to 65472,
 *   or batch 256 with k up to 4032, k being a multiple of 64); larger sizes
 *   return DBF_ERR_WORKSPACE.  The optional areas do not fit, so this call
 *   runs the schedules that need none (no single-launch decode, no stream-K).
 *   The first call on each device looks up the buffer's device address with
 *   that device current; make that first call before any stream capture.  A
 *   failed lookup (DBF_ERR_CUDA) is not remembered: the next call retries.
 *   Device-side failures (a bounded wait that gave up) are read back with
 *   dbf_noalloc_status.
 *   Each call clears the buffer's status word (cudaMemsetAsync on `stream`)
 *   before its kernels; the buffer keeps the last call's other contents.
 *   All calls share the one buffer: calls whose work overlaps on the GPU
 *   (other streams, other host threads) race on it and must be serialised by
 *   the caller.  Argument checks are those of dbf_forward and run first.
 */
DBF_API dbf_status dbf_forward_noalloc(const uint16_t* x, const uint32_t* packedA, const uint32_t* packedB,
                                       const uint16_t* a, const uint16_t* m, const uint16_t* b, int64_t n,
                                       int64_t k, int64_t m_in, int64_t batch, void* y, dbf_dtype y_t,
                                       uint32_t flags, struct CUstream_st* stream);

/*
 * The status word of dbf_forward_noalloc's library buffer on the current
 * device, copied to *device_status (synchronises `stream`): 0 if the last
 * dbf_forward_noalloc call's kernels (the word is cleared at each call) saw
 * no device-side wait give up, else the dbf_status of the first failure
 * (DBF_ERR_TIMEOUT).  Like dbf_forward_noalloc it allocates nothing; its first
 * use on a device looks the buffer up as described there.  (No counterpart
 * in the pages: it reports on the library's own buffer.)
 */
DBF_API dbf_status dbf_noalloc_status(struct CUstream_st* stream, int32_t* device_status);

/*
 * Several layers that read the same input x: the same computation as one
 * dbf_forward per layer (section 2.1, computation process), with the layers'
 * first products in one launch and their second products in another.  The
 * pages evaluate one layer at a time; grouping layers that share their input
 * (a decoder's q, k and v projections, or its gate and up projections) is an
 * engineering choice of this library: at batch 1 each launch costs latency
 * that does not grow with its size, so G layers in two launches cost far less
 * than G layers in 2G.
 *
 *   layers[g]  packedA, packedB, a, m, b: as in dbf_forward for layer g, of
 *              n = layers[g].n rows and middle dimension k = layers[g].k, all
 *              over the shared m_in; y: batch x n output of layer g
 *              (row-major, y_t).  The array is read during the call only.
 *   num_layers 1 .. DBF_MAX_GROUP.
 *   workspace  ws_bytes >= 256 + sum over layers of round_up(batch * k_g * 2,
 *              256); dbf_forward_grouped_workspace_bytes(...) adds the
 *              stream-K area past 128 tokens.  Zero-filled before its first use.
 * Per-layer results equal dbf_forward's up to the order of fp32 additions
 * (the K split can differ); in integer mode they are identical.
 * Shape contract per layer as dbf_forward; flags as dbf_forward.
 */
#define DBF_MAX_GROUP 8
typedef struct dbf_layer_desc {
  const uint32_t* packedA;
  const uint32_t* packedB;
  const uint16_t* a;
  const uint16_t* m;
  const uint16_t* b;
  int64_t n;
  int64_t k;
  void* y;
} dbf_layer_desc;

/* Workspace bytes for dbf_forward_grouped (0 if an argument is out of range):
 * 256 + sum over layers of round_up(batch * k_g * 2, 256), plus past 128
 * tokens the stream-K area of dbf_forward_workspace_bytes (shared by the
 * layers, which run one after another). */
DBF_API size_t dbf_forward_grouped_workspace_bytes(const dbf_layer_desc* layers, int num_layers, int64_t m_in,
                                                   int64_t batch);

DBF_API dbf_status dbf_forward_grouped(const uint16_t* x, int64_t m_in, int64_t batch, const dbf_layer_desc* layers,
                                       int num_layers, dbf_dtype y_t, void* workspace, size_t ws_bytes,
                                       uint32_t flags, struct CUstream_st* stream);

/*
 * Transpose of a packed sign matrix: `packed` holds S (rows x cols) in the
 * packed layout; `out` receives S^T (cols rows over `rows` columns), i.e.
 * dbf_packed_words(cols, rows) words, in the same layout with zero padding.
 * Used to pack A^T and B^T for dbf_forward_transposed without the +-1 matrices.
 * Not a hot path.  Both pointers 16-byte aligned; out must not overlap packed.
 */
DBF_API dbf_status dbf_transpose_signs(const uint32_t* packed, int64_t rows, int64_t cols, uint32_t* out,
                                       struct CUstream_st* stream);

/*
 * The transpose product dx = dy W of the layer of dbf_forward (W is n x m_in,
 * y = x W^T, so this is the input gradient):
 *     dx = b (.) (B^T (m (.) (A^T (a (.) dy))))      (section 2.1 read right to left)
 *   dy         batch x n fp16, row-major.
 *   packedAT   A^T packed: k rows over n   (dbf_transpose_signs of packedA).
 *   packedBT   B^T packed: m_in rows over k (dbf_transpose_signs of packedB).
 *   a, m, b    the layer's scales (n, k, m_in entries), as in dbf_forward.
 *   dx         batch x m_in, dx_t = DBF_F16 or DBF_F32.
 *   workspace  ws_bytes >= dbf_forward_workspace_bytes(m_in, k, n, batch).
 * It is dbf_forward with B^T and A^T as the two factors and a and b
 * exchanged, so the arithmetic (fp32 accumulation, fp16 a (.) dy on the decode
 * path, fp16 middle vector) and the paths are those of dbf_forward.  Shape
 * contract: k and n multiples of 64 in [64, 1 << 20], m_in and batch in
 * [1, 1 << 24].
 */
DBF_API dbf_status dbf_forward_transposed(const uint16_t* dy, const uint32_t* packedAT, const uint32_t* packedBT,
                                          const uint16_t* a, const uint16_t* m, const uint16_t* b, int64_t n,
                                          int64_t k, int64_t m_in, int64_t batch, void* dx, dbf_dtype dx_t,
                                          void* workspace, size_t ws_bytes, uint32_t flags,
                                          struct CUstream_st* stream);

/*
 * Binary Quadratic Quantization (BQQ) forward, on the sign-product kernels.
 * The sciencestack.ai page of "Binary Quadratic Quantization: Beyond
 * First-Order Quantization for Real-Valued Matrix Compression" (TL;DR) writes
 * a compressed n x m_in matrix as
 *     W = sum_{i<p} (r_i Y_i Z_i + s_i Y_i 1_Z + t_i 1_Y Z_i) + u 1
 * with binary Y_i (n x k) and Z_i (k x m_in) and all-ones matrices 1_Z, 1_Y, 1
 * of the shapes of Z_i, Y_i and W.  The binary entries are read as {0, 1}.
 * y = x W^T is evaluated as one DBF product plus a rank-two correction:
 *     y = S_Y diag(r_i / 4 per term) S_Z x + c (1^T x) + 1 (d^T x),
 * S_Y = 1 - 2 [Y_0 .. Y_p-1] and S_Z = 1 - 2 [Z_0; ..; Z_p-1] as sign matrices,
 * c = sum_i (s_i + r_i/2) rowsum(Y_i), d = sum_i (t_i + r_i/2) colsum(Z_i)
 * + u - k sum_i r_i / 4 (exact algebra; no approximation).
 *
 *   packedY    [Y_0 .. Y_{p-1}] side by side, n rows over p*k columns, in the
 *              packed layout with a set bit for each 1 (dbf_pack_signs of
 *              1 - 2Y, or of -Y).
 *   packedZ    [Z_0; ..; Z_{p-1}] stacked, p*k rows over m_in columns, likewise.
 *   r, s, t    p fp16 scalars each; u one fp16 scalar (device pointers).
 *   prepared   dbf_bqq_prepared_bytes(...) bytes, written by dbf_bqq_prepare:
 *              mid = r_i / 4 (p*k fp16), a vector of ones, c (n fp32) and
 *              d (m_in fp32).  It depends on the weights only: prepare once.
 * Shape contract: p*k and m_in multiples of 64 in [64, 1 << 20]; n and batch
 * in [1, 1 << 24]; p <= 4096.  Pointers 16-byte aligned.
 * dbf_bqq_forward: x batch x m_in fp16, y batch x n (y_t DBF_F16 or DBF_F32),
 * workspace >= dbf_bqq_workspace_bytes(...) zero-filled before its first use;
 * flags as dbf_forward.  Arithmetic: the product term as dbf_forward (fp32
 * accumulation), the correction in fp32, one rounding to y_t.
 */
DBF_API size_t dbf_bqq_prepared_bytes(int64_t n, int64_t k, int64_t p, int64_t m_in);
DBF_API dbf_status dbf_bqq_prepare(const uint32_t* packedY, const uint32_t* packedZ, const uint16_t* r,
                                   const uint16_t* s, const uint16_t* t, const uint16_t* u, int64_t n, int64_t k,
                                   int64_t p, int64_t m_in, void* prepared, size_t prepared_bytes,
                                   struct CUstream_st* stream);
DBF_API size_t dbf_bqq_workspace_bytes(int64_t n, int64_t k, int64_t p, int64_t m_in, int64_t batch);
DBF_API dbf_status dbf_bqq_forward(const uint16_t* x, const uint32_t* packedY, const uint32_t* packedZ,
                                   const void* prepared, int64_t n, int64_t k, int64_t p, int64_t m_in, int64_t batch,
                                   void* y, dbf_dtype y_t, void* workspace, size_t ws_bytes, uint32_t flags,
                                   struct CUstream_st* stream);

/*
 * Offline factorisation of a dense weight into the DBF form (gist.science
 * technical summary, section 2.2, optimisation algorithm: alternating
 * minimisation over the two factors, ADMM for each sign-constrained problem,
 * SVID projection onto "sign matrix times rank-one magnitudes").  Not a hot
 * path: it prepares weights once.
 *
 * The factors are dense fp32 matrices in SVID form: L = diag(a) A diag(mL)
 * (n x k) and R = diag(mR) B diag(b) (k x m), W ~= L R.  The caller provides the
 * starting pair (dbf_factorize_start: a random projection of W's range) and
 * runs passes, keeping the best pair; dbf_factorize_finish turns it into the
 * packed signs and fp16 scales that dbf_forward takes.
 *
 * dbf_factorize_pass: one alternating pass, in place on L and R:
 *   left:  G = 2 R R^T + rho I, rho = trace(2 R R^T)/k; Z = L, U = 0;
 *          admm_steps times: L' = (2 W R^T + rho (Z - U)) G^-1,
 *          Z = SVID(L' + U), U += L' - Z;  then L = Z;
 *   right: the same for R with L fixed; then *err = ||W - L R||_F / ||W||_F
 *   (one fp32 in device memory).  A pass need not lower the error: keep the
 *   best pair (the Python binding's dbf_factorize does).
 *   W: n x m fp32 row-major; L: n x k; R: k x m (device, row-major, fp32).
 *   workspace: dbf_factorize_workspace_bytes(n, m, k) bytes of device memory.
 *   Shape: n, m <= 65536, k <= 16384, n*m and k*max(n, m) <= 2^31.
 *   Arithmetic: fp32 (cuBLAS SGEMM for the dense products, no tensor-op math);
 *   G^-1 from a Cholesky factorisation (cuSOLVER potrf / potri; G's
 *   eigenvalues lie in [rho, rho + lambda_max(2 R R^T)], rho their mean, so
 *   it is well conditioned); SVID's magnitudes by 30 power steps on |M|.
 *   Deterministic.  The solver's scratch lives in the workspace when it fits
 *   in 2 k^2 floats, else it is taken from and returned to the stream-ordered
 *   allocator of the current device within the call (small k only).
 * dbf_svid: the leading singular pair of |M| (rows x cols, fp32): unit vectors
 *   u (rows) and v (cols) and sigma (one fp32), all device memory (scratch:
 *   dbf_svid_workspace_bytes(rows, cols) bytes of device workspace), so that
 *   sign(M) (.) (sigma u v^T) is M's SVID projection (a = sqrt(sigma) u,
 *   b = sqrt(sigma) v in the DBF scale vectors).
 */
/* dbf_factorize_start: L = SVID(W Omega) (n x k), R = SVID(Omega^T) (k x m) for a
 *   caller-drawn m x k projection Omega (fp32; e.g. random signs / sqrt(m)), and
 *   *err = the start's relative error.
 * dbf_factorize_finish: the DBF form of a pair in SVID form: packedA / packedB
 *   (dbf_packed_words(n, k) / (k, m) words, a set bit where L / R is negative),
 *   a (n), mid (k), b (m) fp16 with W ~= (a (.) A (.) mid^T)(B (.) b^T). */
DBF_API size_t dbf_factorize_workspace_bytes(int64_t n, int64_t m, int64_t k);
DBF_API dbf_status dbf_factorize_start(const float* W, const float* Omega, int64_t n, int64_t m, int64_t k, float* L,
                                       float* R, float* err, void* workspace, size_t ws_bytes,
                                       struct CUstream_st* stream);
DBF_API dbf_status dbf_factorize_finish(const float* L, const float* R, int64_t n, int64_t m, int64_t k,
                                        uint32_t* packedA, uint32_t* packedB, uint16_t* a, uint16_t* mid, uint16_t* b,
                                        void* workspace, size_t ws_bytes, struct CUstream_st* stream);
DBF_API dbf_status dbf_factorize_pass(const float* W, int64_t n, int64_t m, int64_t k, float* L, float* R,
                                      int admm_steps, float* err, void* workspace, size_t ws_bytes,
                                      struct CUstream_st* stream);
DBF_API size_t dbf_svid_workspace_bytes(int64_t rows, int64_t cols);
DBF_API dbf_status dbf_svid(const float* M, int64_t rows, int64_t cols, float* u, float* v, float* sigma,
                            void* workspace, size_t ws_bytes, struct CUstream_st* stream);

/* Static, NUL-terminated description of a status code. */
DBF_API const char* dbf_status_string(dbf_status status);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* DBF_H_ */
