/*
 * mqv.h -- C ABI of the MicroQonv hot path on NVIDIA B200 (sm_100a).
 *
 * The method (MicroQonv summary, onedev.kr/papers/182):
 *   section "어떻게 동작하나" (how it works): activations are quantized once,
 *     before im2col, and kept in the channel-batch-first layout
 *     X_{Cin,N} in R^{Cin·(Hin·Win·N)}: for every pixel (h, w) the Cin x N
 *     values are one contiguous block, batch index n fastest;
 *   section "무엇과 다른가" (how it differs): W is Cout x (Kh·Kw·Cin), G_Y is
 *     Cout x (Hout·Wout·N); 4 x 4 square blocks (B = 16) so each block side
 *     lies along the contraction of every one of the three GEMMs
 *     Y = W·X', G_W = G_Y·X'^T, G_X' = W^T·G_Y; NVFP4 two-level scales
 *     T = max|X| / (448·emax), B = CastE4M3(blockmax / (T·emax)),
 *     code = Round(x / (B·T)); round-to-nearest for X and W, stochastic
 *     rounding for G_Y;
 *   section "어떻게 쓰나" (how it is used): the NVFP6 variant, E2M3 elements.
 *
 * Conventions for every entry point
 *   - All pointers named src/dst/codes/scales/tscale/y/gw/gx/ws are DEVICE
 *     pointers owned by the caller; the library never allocates, frees or
 *     keeps them.  Descriptor structs are host memory, read during the call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *     Every call only enqueues work on it and returns; nothing synchronizes.
 *   - Arguments are validated before anything is enqueued; on any error the
 *     call returns a non-zero mqv_status, enqueues nothing, and
 *     mqv_last_error() (per host thread) describes the problem.
 *   - fp32 tensors use these layouts (row-major, last index fastest):
 *       X   [H][W][Cin][N]     2D view rows = H·W·Cin,     cols = N
 *       W   [Cout][Kh][Kw][Cin] 2D view rows = Cout,       cols = Kh·Kw·Cin
 *       G_Y [Ho][Wo][Cout][N]  2D view rows = Ho·Wo·Cout,  cols = N
 *       Y   [Ho][Wo][Cout][N], G_X [H][W][Cin][N], G_W [Cout][Kh][Kw][Cin]
 *     with Ho = (H + 2·pad - Kh)/stride + 1 (floor), same for Wo.
 *   - A quantized tensor (mqv_qtensor) of a rows x cols view holds
 *       codes : packed element codes, row-major.  NVFP4: two 4-bit codes per
 *               byte, even column in the low nibble (cols/2 bytes per row).
 *               NVFP6: four 6-bit codes per 3 bytes, code j of a group at
 *               bits [6j, 6j+6) of the little-endian 24-bit word
 *               (3·cols/4 bytes per row).  Code = sign bit | magnitude bits
 *               (E2M1 or E2M3 as in OCP MX v1.0).
 *       scales: one E4M3 byte per 4 x 4 block, [rows/4][cols/4] row-major.
 *       tscale: one fp32 tensor scale T.
 *     A 4 x 4 block of X or G_Y is 4 channels x 4 batch items at one pixel;
 *     of W, 4 output channels x 4 input channels at one tap.
 */
#ifndef MQV_H
#define MQV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MQV_OK = 0,
  MQV_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer    */
  MQV_ERR_UNSUPPORTED = 2,  /* shape/format outside what the kernels handle  */
  MQV_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required    */
  MQV_ERR_CUDA = 4,         /* a CUDA launch or query failed                 */
  MQV_ERR_TIMEOUT = 5       /* a bounded device-side wait gave up            */
} mqv_status;

typedef enum { MQV_NVFP4 = 0 /* E2M1 elements */, MQV_NVFP6 = 1 /* E2M3 */ } mqv_format;
typedef enum { MQV_RNE = 0, MQV_SR = 1 } mqv_rounding;
typedef enum { MQV_OP_FWD = 1, MQV_OP_WGRAD = 2, MQV_OP_DGRAD = 3, MQV_OP_FWD_BLOCKSCALED = 4 } mqv_op;

/* Shape of one convolution layer (the pages' N, Cin, Cout, H, W, Kh, Kw,
 * stride, pad, format).  Requirements: all > 0 (pad >= 0), Cin, Cout and N
 * multiples of 4, pad < Kh and pad < Kw, Ho and Wo >= 1, fmt a mqv_format. */
typedef struct {
  int64_t N, Cin, Cout, H, W, Kh, Kw, stride, pad;
  int32_t fmt;
  int32_t reserved; /* must be 0 */
} mqv_conv_desc;

/* Block shape of a quantized view's scale plane.  MicroQonv's own blocks are
 * the 4 x 4 squares.  The two 16-element line shapes are the plain blocks of
 * the scheme the MicroQonv summary (section "무엇인가") sets it against:
 * after im2col, each GEMM operand is quantized in 16 consecutive elements
 * along that GEMM's contraction, once per direction.
 *   MQV_BLOCKS_4X4   scales [rows/4][cols/4]
 *   MQV_BLOCKS_1X16  16 consecutive columns of one row: scales [rows][cols/16]
 *                    (cols a multiple of 16)
 *   MQV_BLOCKS_16X1  16 consecutive rows of one column: scales [rows/16][cols]
 *                    (rows a multiple of 16)
 * The code plane is the same for all three.  Every entry point takes the
 * square blocks.  mqv_quantize_many and mqv_dequantize take all three.  The
 * conv passes take the line shapes only on the kernels the naive scheme
 * runs on: a stride-1 1 x 1 layer, with the shapes listed at each pass. */
typedef enum { MQV_BLOCKS_4X4 = 0, MQV_BLOCKS_1X16 = 1, MQV_BLOCKS_16X1 = 2 } mqv_blocks;

/* A quantized rows x cols view (see the layout notes above).  codes and
 * scales must be 16-byte aligned device pointers. */
typedef struct {
  void* codes;
  uint8_t* scales;
  float* tscale;
  int64_t rows, cols;
  int32_t fmt;
  int32_t blocks;   /* mqv_blocks; 0 (the 4 x 4 squares) unless stated */
} mqv_qtensor;

/* Library version (major*10000 + minor*100 + patch). */
int32_t mqv_version(void);

/* Message of the last error returned on this host thread ("" if none). */
const char* mqv_last_error(void);

/* Bytes of the packed codes and of the scale plane of a rows x cols view.
 * rows and cols must be positive multiples of 4. Host-only, no CUDA calls. */
mqv_status mqv_qtensor_bytes(int64_t rows, int64_t cols, int32_t fmt,
                             size_t* code_bytes, size_t* scale_bytes);

/* Workspace bytes that mqv_quantize_cbf needs for a rows x cols view
 * (per-CTA partial maxima of |x|).  Host-only. */
mqv_status mqv_quantize_workspace_size(int64_t rows, int64_t cols, size_t* bytes);

/* Quantize once, section "무엇과 다른가": amax = max|src| over the whole
 * view, T = amax / (448·emax) (emax = 6 for NVFP4, 7.5 for NVFP6), per 4 x 4
 * block B = CastE4M3(blockmax / (T·emax)), code = Round(x / (B·T)) with
 * round-to-nearest-even (MQV_RNE) or Philox4x32-10 stochastic rounding
 * (MQV_SR: element i of the row-major view uses word i&3 of counter
 * (i>>2 as two 32-bit words, 0, 0) and key (seed as two 32-bit words);
 * round up iff (word>>8)·2^-24 < fractional position).  Two launches: a
 * |x| max reduction into `ws`, then the block quantizer (which finishes the
 * reduction itself).  src: rows x cols fp32, 16-byte aligned, finite (a NaN
 * or infinity gives unspecified codes, never a fault).  Tiny tensors,
 * subnormal elements included, quantize exactly as defined (blocks whose
 * divisor B·T is below 2^-64 divide with the IEEE divide).  out: codes,
 * scales and tscale written; out->rows/cols/fmt must match. */
mqv_status mqv_quantize_cbf(const float* src, int64_t rows, int64_t cols, int32_t fmt,
                            int32_t rounding, uint64_t seed, const mqv_qtensor* out,
                            void* ws, size_t ws_bytes, void* stream);

/* The reduction step alone: *amax (device fp32) = max|src| of the view.
 * ws: at least mqv_quantize_workspace_size bytes.  Used when the amax of a
 * tensor sharded across processes must be combined (a MAX all-reduce of one
 * float) before quantizing. */
mqv_status mqv_amax(const float* src, int64_t rows, int64_t cols, float* amax,
                    void* ws, size_t ws_bytes, void* stream);

/* The quantize step alone, given a device fp32 amax (from mqv_amax, possibly
 * combined across processes).  Same arithmetic as mqv_quantize_cbf.  For a
 * batch shard the view holds columns [sr_col0, sr_col0 + cols) of a view
 * with sr_cols columns; stochastic rounding then numbers element (r, c) as
 * r·sr_cols + sr_col0 + c, so the shard draws the same Philox words as the
 * whole tensor would (sr_cols = 0 means an unsharded view: sr_cols = cols).
 * sr_col0 must be a multiple of 4. */
mqv_status mqv_quantize_with_amax(const float* src, int64_t rows, int64_t cols,
                                  int32_t fmt, int32_t rounding, uint64_t seed,
                                  const float* amax, int64_t sr_col0, int64_t sr_cols,
                                  const mqv_qtensor* out, void* stream);

/* One tensor of a mqv_quantize_many call: the arguments of mqv_quantize_cbf. */
typedef struct {
  const float* src;
  int64_t rows, cols;
  int32_t fmt, rounding;
  uint64_t seed;
  mqv_qtensor out;
} mqv_quantize_job;

/* Workspace bytes of mqv_quantize_many for these jobs.  Host-only. */
mqv_status mqv_quantize_many_workspace_size(const mqv_quantize_job* jobs, int32_t count,
                                            size_t* bytes);

/* Quantize 1..8 tensors (for a layer: X and W with RNE, G_Y with SR) in two
 * launches: one amax pass over all of them, then one quantize pass.  Each
 * tensor's codes, scales and T are bit-identical to mqv_quantize_cbf on it
 * alone.  jobs: host array; every job is validated as mqv_quantize_cbf's
 * arguments are; outputs must not overlap.  ws: at least
 * mqv_quantize_many_workspace_size bytes, 16-byte aligned. */
mqv_status mqv_quantize_many(const mqv_quantize_job* jobs, int32_t count, void* ws, size_t ws_bytes,
                             void* stream);

/* dst[r][c] = code·B·T of a quantized view, fp32 (code·B is exact in fp16;
 * the product with T is one fp32 rounding).  Reads a stored (for example
 * latent-replay) tensor back.  dst: rows x cols fp32, 16-byte aligned. */
mqv_status mqv_dequantize(const mqv_qtensor* q, float* dst, void* stream);

/* Latent-replay form of a post-ReLU tensor (sections "어떻게 쓰나" and
 * "전제와 한계": an E2M1 activation takes 3 bits per pixel, and the replay
 * buffer keeps quantized activations).  After ReLU no code is negative, so
 * only the magnitude bits are kept, m = 3 (NVFP4) or 5 (NVFP6): element i of
 * the row-major rows x cols view at bits [i·m, i·m + m) of a little-endian
 * bit stream, rows·cols·m/8 bytes.  The scale plane and T are not part of it
 * (keep them as they are).  With the scales that is 3.5 bits per element
 * for NVFP4 and 5.5 for NVFP6.  rows and cols: positive multiples of 4. */
mqv_status mqv_replay_bytes(int64_t rows, int64_t cols, int32_t fmt, size_t* bytes);

/* Write the replay form of q's codes to `packed` (16-byte aligned device
 * buffer of mqv_replay_bytes bytes).  A code with the sign bit and a nonzero
 * magnitude (a negative value) is stored as 0, the ReLU of its value; if
 * `negatives` is not NULL, the number of such codes is added to the device
 * uint32 it points to (the caller zeroes it).  Reads q->codes only. */
mqv_status mqv_replay_pack(const mqv_qtensor* q, void* packed, uint32_t* negatives, void* stream);

/* Codes (standard packing, sign bit 0) of a rows x cols view from its
 * replay form.  packed, codes: 16-byte aligned device buffers. */
mqv_status mqv_replay_unpack(const void* packed, int64_t rows, int64_t cols, int32_t fmt, void* codes,
                             void* stream);

/* Read the replay form straight back to fp32: dst[r][c] = code·B·T with the
 * arithmetic of mqv_dequantize (code·B exact in fp16, one fp32 rounding).
 * scales: [rows/4][cols/4] E4M3 bytes; tscale: one device fp32; dst: rows x
 * cols fp32, 16-byte aligned. */
mqv_status mqv_replay_dequantize(const void* packed, const uint8_t* scales, const float* tscale, int64_t rows,
                                 int64_t cols, int32_t fmt, float* dst, void* stream);

/* Workspace bytes for a conv pass (op = mqv_op).  Host-only. */
mqv_status mqv_conv_workspace_size(const mqv_conv_desc* d, int32_t op, size_t* bytes);

/* Forward GEMM Y = W·X' (section "무엇과 다른가"), implicit: im2col rows of
 * X' are gathered from the quantized X on chip, never stored.
 * y[ho][wo][co][n] = T_w·T_x·sum_{kh,kw,ci} Wq[co][kh][kw][ci]·Xq[hi][wi][ci][n]
 * with hi = ho·stride + kh - pad, wi = wo·stride + kw - pad, zero outside.
 * w: view Cout x Kh·Kw·Cin; x: view H·W·Cin x N; y fp32 [Ho][Wo][Cout][N].
 * Block shapes: both operands 4 x 4, or, on a stride-1 1 x 1 layer with
 * N a multiple of 16, w in MQV_BLOCKS_1X16 and x in MQV_BLOCKS_16X1 (the
 * naive scheme's blocks along the contraction K). */
mqv_status mqv_conv_fwd(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* x,
                        float* y, void* ws, size_t ws_bytes, void* stream);

/* The forward pass of mqv_conv_fwd on the other MMA form sm_100a offers for
 * these operands: the native block-scaled MMA (tcgen05.mma kind::mxf4nvf4,
 * E2M1 operands with one UE4M3 scale per 16 consecutive K elements).  Section
 * "무엇과 다른가" gives each 4 x 4 square block one E4M3 scale, i.e. 4 K
 * elements per scale in every row, so the only exact mapping pads each
 * 4-element block row with 12 zero codes: the codes enter the MMA without
 * dequantization, the block scales travel in tensor memory, and 3/4 of the
 * MMA's K is zeros.  Kept beside mqv_conv_fwd (fp16 products of dequantized
 * operands, exact) so the two forms can be measured on the same layer; the
 * outputs agree within the parity tolerance (both accumulate exact products
 * in fp32, in different orders).  Supported: NVFP4, stride 1, N = 64 or
 * 128 with (128/N + Kw - 1)·N <= 256, Kw <= 3, Cin a multiple of 64; other
 * layers return MQV_ERR_UNSUPPORTED before any launch.  ws:
 * mqv_conv_workspace_size(d, MQV_OP_FWD_BLOCKSCALED) bytes (the padded
 * weight image and its scales); other arguments as mqv_conv_fwd. */
mqv_status mqv_conv_fwd_blockscaled(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* x,
                                    float* y, void* ws, size_t ws_bytes, void* stream);

/* Weight-gradient GEMM G_W = G_Y·X'^T: contraction over (ho, wo, n), split
 * across CTAs and summed in a fixed order (deterministic) through `ws`.
 * gy: view Ho·Wo·Cout x N; x: view H·W·Cin x N; gw fp32 [Cout][Kh][Kw][Cin].
 * Block shapes: both 4 x 4, or, on a stride-1 1 x 1 layer, both
 * MQV_BLOCKS_1X16 (blocks along the contraction over (ho, wo, n)). */
mqv_status mqv_conv_wgrad(const mqv_conv_desc* d, const mqv_qtensor* gy, const mqv_qtensor* x,
                          float* gw, void* ws, size_t ws_bytes, void* stream);

/* Weight gradient exactly as mqv_conv_wgrad (same split plan, same
 * results), for callers that cannot allocate device memory at all: code
 * that runs where every byte of device memory is owned by someone else's
 * fixed pool (an inference server or framework plugin that may not grow its
 * footprint), or that has no allocator to ask for a workspace.  The paper
 * has no counterpart; this is an interface convenience of this library.
 *   - Allocates nothing: the split-K partial sums go to one file-scope
 *     device array of 32 MiB inside the library, which every GPU that loads
 *     the library holds until the process exits.  Layers whose partials
 *     would need more (mqv_conv_workspace_size(d, MQV_OP_WGRAD) > 32 MiB)
 *     are rejected with MQV_ERR_UNSUPPORTED and a message; the current split
 *     planner stays below 29.1 MB for every shape.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents;
 *     every partial a call reads was written by the same call, so nothing
 *     needs clearing.  Calls that overlap on the GPU (other streams, other
 *     host threads) race on the array: serialize them.
 * gy, x, gw and stream as in mqv_conv_wgrad. */
mqv_status mqv_conv_wgrad_noalloc(const mqv_conv_desc* d, const mqv_qtensor* gy,
                                  const mqv_qtensor* x, float* gw, void* stream);

/* Input-gradient G_X = col2im(W^T·G_Y), computed directly as an implicit
 * transposed convolution: gx[hi][wi][ci][n] = T_w·T_g·sum over (kh, kw, co)
 * and every (ho, wo) with ho·stride + kh - pad = hi, wo·stride + kw - pad = wi.
 * w: view Cout x Kh·Kw·Cin; gy: view Ho·Wo·Cout x N; gx fp32 [H][W][Cin][N].
 * Block shapes: both 4 x 4, or, on a stride-1 1 x 1 layer with N a
 * multiple of 16, both MQV_BLOCKS_16X1 (blocks along the contraction over
 * Cout). */
mqv_status mqv_conv_dgrad(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* gy,
                          float* gx, void* ws, size_t ws_bytes, void* stream);

/* Forward pass with the next quantization's first step fused into its
 * epilogue.  Quantize-once needs the global max|x| of a tensor before any
 * block can be scaled (section "무엇과 다른가": T = max|X| / (448·emax)); the
 * tensor the next layer quantizes is this pass's output, so the epilogue
 * that writes it can also reduce it, and the separate max pass (a full fp32
 * read) disappears.  Outputs as mqv_conv_fwd, plus:
 *   relu   0: y as mqv_conv_fwd; 1: y = max(conv, 0) (-0 and NaN become +0),
 *          the next layer's post-ReLU input X.
 *   y_amax NULL, or a device fp32 that receives max|y| over the stored
 *          values (exactly what mqv_amax of y would return).  The call
 *          enqueues a 4-byte clear of it, then the kernels' atomic updates;
 *          read it after the stream reaches that point.  Feed it to
 *          mqv_quantize_with_amax to quantize y in one pass with codes
 *          bit-identical to mqv_quantize_cbf of y. */
mqv_status mqv_conv_fwd_fused(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* x, float* y,
                              int32_t relu, float* y_amax, void* ws, size_t ws_bytes, void* stream);

/* Input-gradient pass with max|gx| fused into its epilogue (gx_amax as
 * y_amax above); gx is the G_Y of the layer before, which the backward pass
 * quantizes next with stochastic rounding. */
mqv_status mqv_conv_dgrad_fused(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* gy, float* gx,
                                float* gx_amax, void* ws, size_t ws_bytes, void* stream);

/* The forward pass writing the next layer's quantized input instead of
 * fp32 Y (section "어떻게 동작하나": Y comes out in the channel-batch-first
 * layout the next layer consumes, so the epilogue can quantize it in place
 * and the fp32 round trip through HBM disappears).  Quantize-once needs T
 * before any block can be scaled, and a tile's epilogue runs before the
 * whole output exists, so T comes from a given max |x|: t_amax, a device
 * fp32, for example max|Y| of the previous step (delayed scaling; the call
 * reports this step's max in y_amax).  With t_amax equal to max|Y| of this
 * output the codes, scales and T are exactly those of mqv_quantize_cbf on
 * the fp32 Y (after ReLU when relu = 1) that mqv_conv_fwd_fused stores;
 * with another value they are those of mqv_quantize_with_amax given it
 * (values above it saturate).  Round to nearest (the activations' rule).
 *   y_q    the next layer's X: a view of Ho·Wo·Cout rows x N, d->fmt;
 *          codes, scales and tscale written (nothing in fp32).
 *   relu, y_amax  as mqv_conv_fwd_fused (y_amax NULL or a device fp32).
 * Stride-1 layers of the kernel-row path (N divides 256, N % 8 == 0, Cin a
 * multiple of 64); other layers return MQV_ERR_UNSUPPORTED. */
mqv_status mqv_conv_fwd_quantized(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* x,
                                  int32_t relu, const float* t_amax, const mqv_qtensor* y_q, float* y_amax,
                                  void* ws, size_t ws_bytes, void* stream);

/* The input-gradient pass writing G_X quantized as the next (earlier)
 * layer's G_Y, with Philox stochastic rounding (the gradients' rule; element
 * (r, c) of the H·W·Cin x N view draws word (r·N + c) & 3 of counter
 * (r·N + c) >> 2 with key `seed`, as mqv_quantize_cbf) and T from t_amax as
 * above; gx_amax NULL or a device fp32 that receives max|G_X|.  Stride-1
 * layers of the kernel-row path (Cout a multiple of 64). */
mqv_status mqv_conv_dgrad_quantized(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* gy,
                                    const float* t_amax, uint64_t seed, const mqv_qtensor* gx_q, float* gx_amax,
                                    void* ws, size_t ws_bytes, void* stream);

/* The baseline the method removes (section "무엇인가": quantize after the
 * im2col expansion, once per GEMM direction), for measuring it on the same
 * kernels.  Explicit im2col of fp32 X [H][W][Cin][N] into
 *   xc[(ho, wo)][(kh, kw, ci)][n] = X[ho·stride + kh - pad][wo·stride + kw - pad][ci][n]
 * (zero outside), i.e. fp32 [Ho][Wo][Kh·Kw·Cin][N]: the channel-batch-first
 * tensor of a 1 x 1 convolution with Kh·Kw·Cin input channels whose forward
 * pass is Y = W·X'.  x, xc: 16-byte aligned device buffers the caller owns;
 * xc holds Ho·Wo·Kh·Kw·Cin·N floats (below 2^33).  Asynchronous on stream. */
mqv_status mqv_im2col(const mqv_conv_desc* d, const float* x, float* xc, void* stream);

/* The adjoint of mqv_im2col (reading R14): gx[hi][wi][ci][n] = sum, over
 * the taps (kh, kw) and output pixels (ho, wo) with ho·stride + kh - pad = hi
 * and wo·stride + kw - pad = wi, of gc[(ho, wo)][(kh, kw, ci)][n], added in
 * (kh, kw) order.  gc: fp32 [Ho][Wo][Kh·Kw·Cin][N]; gx: fp32 [H][W][Cin][N]. */
mqv_status mqv_col2im(const mqv_conv_desc* d, const float* gc, float* gx, void* stream);

/* ---- Depthwise layers in BF16 (section "전제와 한계": the pages keep the
 * depthwise convolutions in BF16, outside quantize-once).  One Kh x Kw
 * filter per channel (groups = C), stride and zero padding as for
 * mqv_conv_desc.  Operands are bfloat16 bit patterns (uint16, round to
 * nearest even from fp32 is the caller's conversion): w [C][Kh][Kw], x and
 * gx [H][W][C][N], y and gy [Ho][Wo][C][N]; outputs are fp32.  Products are
 * summed with fp32 FMAs in a fixed order, so results repeat run to run.
 * Validation: sizes positive, N % 4 == 0, stride >= 1, 0 <= pad < Kh, Kw,
 * every tensor below 2^31 elements, pointers 16-byte aligned device
 * memory the caller owns; failures return before anything is launched.
 * Asynchronous on `stream`. */
typedef struct {
  int64_t N, C, H, W, Kh, Kw, stride, pad;
  int32_t reserved; /* must be 0 */
  int32_t reserved2; /* must be 0 */
} mqv_dw_desc;

/* y[ho][wo][c][n] = sum_{kh,kw} w[c][kh][kw]·x[ho·stride+kh-pad][wo·stride+kw-pad][c][n]. */
mqv_status mqv_dw_fwd(const mqv_dw_desc* d, const void* w, const void* x, float* y, void* stream);

/* gx, the adjoint of mqv_dw_fwd in x: gx[hi][wi][c][n] = sum over the taps
 * whose output pixel exists of w[c][kh][kw]·gy[ho][wo][c][n]. */
mqv_status mqv_dw_dgrad(const mqv_dw_desc* d, const void* w, const void* gy, float* gx, void* stream);

/* Workspace bytes of mqv_dw_wgrad (the partial sums of its (ho, wo) parts:
 * for 3x3 filters at stride 1 or 2 one per spatial tile of the output, 8
 * pixels wide; otherwise one per range of output pixels).  Host-only. */
mqv_status mqv_dw_wgrad_workspace_size(const mqv_dw_desc* d, size_t* bytes);

/* gw[c][kh][kw] = sum_{ho,wo,n} gy[ho][wo][c][n]·x[ho·stride+kh-pad][wo·stride+kw-pad][c][n]:
 * partial sums over spatial tiles (or ranges) of output pixels into ws, then
 * added in a fixed order.  ws: at least mqv_dw_wgrad_workspace_size bytes. */
mqv_status mqv_dw_wgrad(const mqv_dw_desc* d, const void* gy, const void* x, float* gw, void* ws,
                        size_t ws_bytes, void* stream);

/* Synchronizes `stream`, then reports and clears the device error word that
 * bounded waits inside the conv kernels set when they give up
 * (*flags = 0: none).  Returns MQV_ERR_TIMEOUT if a flag was set.  Bits:
 * 1 a wait for a free pipeline stage, 2 a wait for a filled stage, 4 a wait
 * for a finished accumulator, 8 the wait of mqv_selftest_wait_timeout.
 * Every such wait polls its mbarrier for about 2^32 SM cycles (about two
 * seconds) before it gives up; the kernel then returns without faulting, so
 * the CUDA context stays usable. */
mqv_status mqv_device_errors(uint32_t* flags, void* stream);

/* Test hook for the timeout path: one CTA waits, with the conv kernels'
 * bounded wait, on an mbarrier that nothing ever arrives at, for at most
 * limit_cycles SM cycles (1 .. 2^32), then sets bit 8 of the device error
 * word and returns.  Nothing else is touched; mqv_device_errors then returns
 * MQV_ERR_TIMEOUT with that bit.  Not part of the method. */
mqv_status mqv_selftest_wait_timeout(int64_t limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MQV_H */
