/*
 * ss2d.h -- C ABI of libss2d, the B200 (sm_100a) SS2D forward core.
 *
 * The operation is the core of the SS2D module in "Deep dive into the SS2D
 * module of VMamba, from theory to code" (section 3, forward_corev0):
 *
 *   CrossScan  (section 3.1, direction table in section 4)
 *       xs[b,k,d,l] = x[b,d,pi_k(l)],  L = H*W,  p = h*W + w,
 *       pi_0(l) = l                       (row-major, left to right)
 *       pi_1(l) = (l mod H)*W + l / H     (column-major, top to bottom)
 *       pi_2(l) = L-1-l                   (reverse of 0)
 *       pi_3(l) = pi_1(L-1-l)             (reverse of 1)
 *   projections (section 3.2, optional)
 *       x_dbl[b,k,c,l] = sum_d x_proj_weight[k,c,d] xs[b,k,d,l]
 *       dts, Bs, Cs = split(x_dbl, [R, N, N]);  dts = dt_projs_weight[k] . dts
 *   selective scan (section 3.2 call with delta_softplus)
 *       delta = softplus(dt + dt_bias[c]),  A = -exp(A_log[c,n])
 *       h_l[n] = exp(delta A[n]) h_{l-1}[n] + delta B_l[n] u_l,   h_{-1} = 0
 *       y_l = sum_n C_l[n] h_l[n] + D[c] u_l
 *   CrossMerge (section 3.3)
 *       y[b,d,p] = y_0[pi_0^-1 p] + y_2[pi_2^-1 p] + y_1[pi_1^-1 p] + y_3[pi_3^-1 p]
 *
 * Conventions shared by every entry point:
 *   - All tensors are dense, row-major, in device memory owned by the caller.
 *     The library never allocates device memory and never synchronises the
 *     device (the one exception is ss2d_device_status, a diagnostic that waits
 *     for its stream); work is enqueued on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream) and runs asynchronously.
 *   - Every tensor pointer must be 16-byte aligned; otherwise the call returns
 *     SS2D_ERR_MISALIGNED and enqueues nothing.
 *   - Arguments are checked on the host before anything is enqueued.  A
 *     failed check returns its status and leaves all buffers untouched.
 *     A failed launch returns SS2D_ERR_CUDA.  The text of the last failure
 *     of the calling thread is available from ss2d_last_error().
 *   - There is no CPU fallback: every entry point runs CUDA kernels built for
 *     sm_100a only.
 */
#ifndef SS2D_H
#define SS2D_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SS2D_OK = 0,
    SS2D_ERR_INVALID_ARG = 1,  /* null pointer, non-positive or inconsistent size */
    SS2D_ERR_UNSUPPORTED = 2,  /* dtype code or state size N outside what is built */
    SS2D_ERR_MISALIGNED = 3,   /* a tensor pointer not 16-byte aligned */
    SS2D_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required */
    SS2D_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed */
    SS2D_ERR_DEVICE = 6        /* a kernel's bounded wait ran out (ss2d_device_status) */
} ss2d_status;

/* Element type codes of the tensors that accept more than one type. */
typedef enum { SS2D_F32 = 0, SS2D_BF16 = 1 } ss2d_dtype;

/* Layouts of the fused core's x and y. */
typedef enum { SS2D_CHANNELS_FIRST = 0, SS2D_CHANNELS_LAST = 1 } ss2d_layout;

/* Static text naming a status code ("SS2D_OK", ...). Never NULL. */
const char *ss2d_status_string(int status);

/* Message of the last failed call on the calling thread ("" if none). */
const char *ss2d_last_error(void);

/* ABI version of this header (major*100 + minor): 101 adds ss2d_core_args.layout,
 * 102 ss2d_core_args.y_dtype, 103 the projection form's backward
 * (ss2d_core_grads.dx_proj_weight and ddt_projs_weight), 104 ss2d_core_args.ckpt,
 * 105 ss2d_device_status and SS2D_ERR_DEVICE, 106 ss2d_core_args.merge_order,
 * 107 the SS2D block (ss2d_block_args, ss2d_block_forward). */
int ss2d_version(void);

/* CrossScan, section 3.1 of the SS2D article.
 * x  : (B, D, H, W), element type `dtype` (SS2D_F32 or SS2D_BF16).
 * xs : (B, 4, D, H*W), same element type; receives x[b,d,pi_k(l)].
 * A pure permutation: the result is bit-identical to the input values. */
int ss2d_cross_scan(const void *x, int dtype, void *xs, int B, int D, int H, int W, void *stream);

/* CrossMerge, section 3.3 of the SS2D article.
 * ys : (B, 4, D, H*W) fp32, the four directions' outputs in scan order.
 * y  : (B, D, H, W) fp32; y[b,d,p] = ((ys0 + flip ys2) + untransposed ys1)
 *      + untransposed flip ys3, added in that order (deterministic). */
int ss2d_cross_merge(const float *ys, float *y, int B, int D, int H, int W, void *stream);

/* Selective scan over C independent channels (the selective_scan call of
 * section 3.2 of the SS2D article, with A passed as A_log).
 * u, delta   : (B, C, L), element types u_dtype / delta_dtype (F32 or BF16).
 * A_log      : (C, N) fp32; A = -exp(A_log).
 * Bm, Cm     : (B, G, N, L) fp32; channel c uses group c / (C/G).  C % G == 0.
 * Dv         : (C) fp32 skip weights, or NULL for D = 0.
 * delta_bias : (C) fp32, or NULL for zero bias.
 * delta_softplus : nonzero applies softplus to delta + bias.
 * y          : (B, C, L) fp32 output; must not alias any input.
 * N must be one of 1, 2, 4, 8, 16.  Results are deterministic. */
int ss2d_selective_scan(const void *u, int u_dtype, const void *delta, int delta_dtype,
                        const float *A_log, const float *Bm, const float *Cm,
                        const float *Dv, const float *delta_bias, int delta_softplus,
                        float *y, int B, int C, int G, int N, int L, void *stream);

/* ss2d_selective_scan with state passing: the scan starts from h0 instead of
 * zero and returns the state after its last step, so that a long sequence can
 * be scanned in consecutive pieces (the chunked recursion of the VSSD article,
 * section 5.2): scanning [0, m) and then [m, L) with h0 = the first call's
 * h_last gives the scan of [0, L).
 *   h0     : (B, C, N) fp32 initial state h_{-1}, or NULL for zero.
 *   h_last : (B, C, N) fp32 output, the state after step L-1, or NULL.
 *   others : as ss2d_selective_scan.
 * h_last must not overlap y or any input; h0 must not overlap y or h_last. */
int ss2d_selective_scan_state(const void *u, int u_dtype, const void *delta, int delta_dtype,
                              const float *A_log, const float *Bm, const float *Cm,
                              const float *Dv, const float *delta_bias, int delta_softplus,
                              const float *h0, float *h_last, float *y,
                              int B, int C, int G, int N, int L, void *stream);

/* Arguments of the fused forward core.  Set struct_size = sizeof(ss2d_core_args).
 * Exactly one of the two parameter sources must be given:
 *   (a) dts, Bs, Cs                      -- the scan inputs directly, or
 *   (b) x_proj_weight, dt_projs_weight   -- the per-direction projections of
 *       section 3.2, computed from x inside the call (needs a workspace). */
typedef struct ss2d_core_args {
    size_t struct_size;
    int B, D, H, W;      /* x is (B, D, H, W); L = H*W */
    int N;               /* state size: 1, 2, 4, 8 or 16 */
    int R;               /* dt_rank (source (b) only; ignored for (a)) */
    const void *x;       /* (B, D, H, W) */
    int x_dtype;         /* SS2D_F32 or SS2D_BF16 */
    const void *dts;     /* (a): (B, 4, D, L) in scan order, or NULL */
    int dts_dtype;       /* (a): SS2D_F32 or SS2D_BF16 */
    const float *Bs;     /* (a): (B, 4, N, L) fp32 in scan order, or NULL */
    const float *Cs;     /* (a): (B, 4, N, L) fp32 in scan order, or NULL */
    const float *A_logs; /* (4*D, N) fp32, channel c = k*D + d */
    const float *Ds;     /* (4*D) fp32, or NULL for D = 0 */
    const float *dt_bias;/* (4*D) fp32, or NULL for zero bias */
    int delta_softplus;  /* nonzero: delta = softplus(dt + dt_bias) */
    const void *x_proj_weight;     /* (b): (4, R+2N, D) bf16, or NULL */
    const float *dt_projs_weight;  /* (b): (4, D, R) fp32, or NULL */
    void *y;             /* (B, D, H, W) output of type y_dtype; must not alias any input */
    int layout;          /* SS2D_CHANNELS_FIRST: x and y are (B, D, H, W) (the default);
                            SS2D_CHANNELS_LAST: x and y are (B, H, W, D), the page's
                            channel_first=False layout -- either form, N = 16, x and
                            dts both bf16 or both fp32, softplus on, D * sizeof(x) a
                            multiple of 16 bytes.  Where a channels-first copy of x is
                            made (the projection form's x_proj GEMM, the backward),
                            ceil(H*W/32) * ceil(D/32) must not exceed 65535.  Callers
                            built against the struct without this field (struct_size =
                            offsetof(ss2d_core_args, layout)) get SS2D_CHANNELS_FIRST. */
    int y_dtype;         /* SS2D_F32 (the default) or SS2D_BF16: the element type of y.  A
                            bf16 y is the fp32 result rounded to nearest even; the four
                            directions are summed in fp32 in the workspace first.  Callers
                            built without this field get SS2D_F32. */
    float *ckpt;         /* NULL, or a (B, 4*D, ceil(L/16), 16) fp32 buffer (16-byte aligned,
                            not overlapping any other tensor) for the scan's checkpoints: the
                            state of every channel before every 16th step.  ss2d_forward_core
                            writes them (dts/Bs/Cs form, N = 16, softplus on, x and dts both
                            bf16 or both fp32, either layout); ss2d_forward_core_backward,
                            called with the same arguments after that forward, reads them
                            instead of recomputing them.  Their order within the buffer is
                            private to the library.  Callers built without this field get
                            NULL. */
    int merge_order;     /* SS2D_MERGE_ATOMIC (the default): the four directions' outputs are
                            added into y with fp32 atomics as each direction's scan produces
                            them, so the order of the four additions, and hence the last bit
                            of y, can differ from run to run.
                            SS2D_MERGE_PAGE_ORDER: y = ((y0 + y2) + y1) + y3 in that order,
                            the association of the SS2D article's section 3.3 (y0 + inv_y0 +
                            wh_y + invwh_y), bit for bit the same on every run: every
                            direction stores its output once, without atomics, into the
                            workspace (channel-first y: the four outputs in scan order, as
                            ss2d_selective_scan writes them; channels-last y: direction 0 into
                            y, the others into three copies of y), and one pass then adds them
                            in that order (ss2d_cross_merge's, for channel-first y).  The
                            workspace grows by 4 (channels-last: 3) * B*D*H*W floats.
                            dts/Bs/Cs form with
                            N = 16, softplus on and x and dts both bf16 or both fp32 only.
                            Callers built without this field get SS2D_MERGE_ATOMIC. */
} ss2d_core_args;

/* Values of ss2d_core_args.merge_order. */
#define SS2D_MERGE_ATOMIC 0
#define SS2D_MERGE_PAGE_ORDER 1

/* Bytes of device workspace ss2d_forward_core needs for these arguments
 * (0 if none).  Returns (size_t)-1 if the arguments are invalid.  y is not
 * read and may be NULL here (y_dtype still counts). */
size_t ss2d_forward_core_workspace(const ss2d_core_args *args);

/* The fused SS2D forward core (forward_corev0 of the SS2D article, section 3,
 * channel-first input, channel-first fp32 output).  The four scan orders are
 * read from x by index arithmetic (xs is never materialised) and each
 * direction's scan output is added into y at the pixel it came from.
 * workspace : device buffer of at least ss2d_forward_core_workspace(args)
 *             bytes (may be NULL when that is 0); contents need not be
 *             initialised and are overwritten.
 * Where the column-major orders read a plane-transposed copy of channels-first
 * x (16-byte aligned rows, N = 16, softplus on), that copy is made in one launch
 * of at most 65535 tiles of 32x32 pixels: a shape with
 * ceil(H/32) * ceil(W/32) > 65535 then returns SS2D_ERR_UNSUPPORTED.
 * The four per-pixel contributions are added with atomics, so the order of
 * those four fp32 additions (and hence the last bit of y) can differ from
 * run to run; everything else is deterministic. */
int ss2d_forward_core(const ss2d_core_args *args, void *workspace, size_t workspace_bytes, void *stream);

/* Gradients of the fused core (the backward of ss2d_forward_core).
 * Set struct_size = sizeof(ss2d_core_grads); the size without the last two members
 * (ABI 102) is still accepted for the dts/Bs/Cs form.  All fp32, dense, 16-byte
 * aligned, in device memory owned by the caller; no gradient may overlap an input
 * or another gradient.  Accumulated gradients are set to zero by the call first,
 * so every output holds exactly the gradient of this call.
 * In the projection form, dts, Bs and Cs are intermediates (the outputs of dt_proj
 * and x_proj, in scan order): ddts, dBs and dCs may then be NULL, and when given
 * they receive the gradients of those intermediates. */
typedef struct ss2d_core_grads {
    size_t struct_size;
    const float *dy;     /* (B, D, H, W): gradient of the loss with respect to y (input) */
    float *dx;           /* (B, D, H, W) */
    float *ddts;         /* (B, 4, D, L), in scan order like dts */
    float *dA_logs;      /* (4D, N), summed over the batch */
    float *dBs;          /* (B, 4, N, L), summed over each direction's D channels */
    float *dCs;          /* (B, 4, N, L), summed over each direction's D channels */
    float *dDs;          /* (4D), summed over the batch, or NULL to skip */
    float *ddt_bias;     /* (4D), summed over the batch, or NULL to skip */
    float *dx_proj_weight;   /* (4, R+2N, D), projection form only (NULL otherwise) */
    float *ddt_projs_weight; /* (4, D, R), projection form only (NULL otherwise) */
} ss2d_core_grads;

/* Bytes of device workspace ss2d_forward_core_backward needs for these forward
 * arguments (args->y is not used and may be NULL).  Returns (size_t)-1 if the
 * arguments are invalid or have no backward (see below). */
size_t ss2d_forward_core_backward_workspace(const ss2d_core_args *args);

/* Reverse-mode gradient of ss2d_forward_core for the loss whose gradient with
 * respect to y is grads->dy: the chain rule applied to the selective-scan
 * recurrence of section 3.2 of the SS2D article (the discrete SSM of the DAMamba
 * article, section 2.1), with CrossScan and CrossMerge (sections 3.1 and 3.3) as
 * each other's adjoints.  The forward is recomputed from per-16-step state
 * checkpoints written into the workspace, and the adjoint state is carried from
 * the last step to the first.
 *   args      : the forward arguments (args->y is not used).  Supported: N <= 16
 *               (below 16 the work is that of 16 states: the state dimension is
 *               padded with inert states in the workspace), softplus on, any
 *               H*W, either layout (with channels-last x,
 *               dy and dx are (B, H, W, D) and the backward runs on channels-first
 *               copies made in the workspace), and either
 *                 - the dts/Bs/Cs form with x and dts both bf16 or both fp32
 *                   (bf16 inputs are widened to fp32 in the workspace), or
 *                 - the projection form (N = 16, bf16 x and x_proj_weight, fp32
 *                   dt_projs_weight, 1 <= R <= 64, D % 16 == 0, B <= 16383): x_proj is
 *                   recomputed on the tensor cores, dt_proj materialised in fp32,
 *                   and the gradients of both projections (section 3.2) follow the
 *                   scan's backward: dx gains the x_proj path, and dx_proj_weight
 *                   and ddt_projs_weight are written.
 *               The planes of x and dy are transposed in one launch each, so
 *               ceil(H/32) * ceil(W/32) may not exceed 65535.
 *               Anything else returns SS2D_ERR_UNSUPPORTED and enqueues nothing.
 *   grads     : dy in, the gradients out (see ss2d_core_grads).  Required: dy, dx,
 *               dA_logs, and ddts, dBs, dCs (dts/Bs/Cs form) or dx_proj_weight and
 *               ddt_projs_weight (projection form).
 *   workspace : at least ss2d_forward_core_backward_workspace(args) bytes,
 *               16-byte aligned, contents need not be initialised.
 * Every gradient is computed in fp32.  dx, dA_logs, dBs, dCs, dDs, ddt_bias and
 * the weight gradients are sums of fp32 atomics, so their last bits can differ
 * from run to run; ddts is deterministic. */
int ss2d_forward_core_backward(const ss2d_core_args *args, const ss2d_core_grads *grads, void *workspace,
                               size_t workspace_bytes, void *stream);

/* Size of the static scratch array of ss2d_forward_core_static (16 MiB). */
#define SS2D_STATIC_SCRATCH_BYTES (16u << 20)

/* The projection form of ss2d_forward_core without a caller-provided
 * workspace.  The pages have no counterpart of this entry point: it exists for
 * callers that cannot allocate device memory at call time -- runtimes and
 * plugin hosts that reserve all device memory up front and forbid allocation
 * on the request path, and code that must not make an allocating (and
 * device-synchronising) call such as cudaMalloc.  It allocates nothing and
 * calls no allocating routine: its scratch is a file-scope device array of
 * SS2D_STATIC_SCRATCH_BYTES that every GPU which loads the library holds until
 * the process exits.
 *   args   : as for ss2d_forward_core, projection form only (x_proj_weight and
 *            dt_projs_weight set, bf16 x); the dts/Bs/Cs form needs no scratch
 *            and returns SS2D_ERR_UNSUPPORTED here.
 *   stream : cudaStream_t on which the work is enqueued (NULL = legacy default).
 * The batch is processed in slices of as many images as fit in the array,
 * one after another on `stream`.  If a single image needs more scratch than
 * the array holds, the call returns SS2D_ERR_UNSUPPORTED with the sizes in
 * ss2d_last_error() and enqueues nothing.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call shares the one array and leaves the last call's
 * contents in it: calls that overlap on the GPU (other streams, other host
 * threads) race on it, so serialise them. */
int ss2d_forward_core_static(const ss2d_core_args *args, void *stream);

/* Device-side status of the projection form's last call on a workspace.
 * The projection form's tensor-core kernels (the x_proj GEMM of the forward
 * and of the backward, and the backward's two x_proj adjoint GEMMs) wait for
 * their MMAs on mbarriers with an iteration limit.  A wait that runs out sets an
 * error word at a fixed place in the workspace, releases the kernel's tensor
 * memory and returns, so the CUDA context stays usable; the outputs of that
 * call are then not valid.  Every projection-form call clears the word before
 * its first tensor-core kernel (ss2d_forward_core_static once per call, not per
 * slice), so it holds the state of the latest call.  This function reads it.
 *   args      : the arguments of that call (they place the word; y is not read).
 *   workspace : the workspace given to that call, or NULL after
 *               ss2d_forward_core_static (its static scratch).
 *   backward  : 0 after ss2d_forward_core or ss2d_forward_core_static,
 *               1 after ss2d_forward_core_backward.
 *   stream    : the call's stream.
 * Returns SS2D_OK or SS2D_ERR_DEVICE.  Unlike every other entry point it
 * synchronises `stream` (a 4-byte device-to-host copy), so it cannot be
 * captured into a CUDA graph.  The dts/Bs/Cs form has no such wait: for it the
 * call returns SS2D_OK without touching the device.  Arguments the matching
 * call would reject return the same status; a NULL workspace with
 * backward = 1 returns SS2D_ERR_WORKSPACE. */
int ss2d_device_status(const ss2d_core_args *args, const void *workspace, int backward, void *stream);

/* ---- The SS2D block around the core (ABI 107) ----------------------------------------
 * The SS2D article (section 1) builds the block from an input projection to the wider
 * D = d_inner channels, a depthwise convolution for local spatial features, the cross
 * scan with the selective scan, and an output projection back to d_model; the VMamba
 * overview page (section 2.2, the SS2D constructor) gives the SiLU activation, the
 * convolution's size d_conv = 3 and a learnable gate on the information flow.  The pages
 * print no forward pass for the block; this one computes, per image, channels last:
 *   xz  = x @ in_proj_weight^T (+ in_proj_bias)          (B, H, W, 2D), stored bf16
 *   x_c = SiLU(depthwise_conv(xz[..., :D]) + conv_bias)  d_conv x d_conv kernel per channel,
 *                                                        zero padding (d_conv - 1) / 2,
 *                                                        stored bf16
 *   y   = the fused core on x_c, projection form (x_proj_weight, dt_projs_weight,
 *         dt_projs_bias as the core's dt_bias, A_logs, Ds, softplus on)     fp32
 *   g   = LayerNorm over D(y) * SiLU(xz[..., D:])        mean and biased variance of each
 *                                                        pixel, eps inside the square root,
 *                                                        stored bf16
 *   out = g @ out_proj_weight^T (+ out_proj_bias)        (B, H, W, d_model)
 * The first D channels of xz feed the scan and the last D the gate.  The two
 * projections run on the tensor cores (bf16 operands, fp32 accumulation). */
typedef struct ss2d_block_args {
    size_t struct_size;            /* sizeof(ss2d_block_args) */
    int B, H, W;                   /* images and their size; L = H*W */
    int d_model;                   /* block channels: a multiple of 16 */
    int D;                         /* d_inner, the core's channels: a multiple of 16, the
                                      LayerNorm tile needs D <= 1648 */
    int N;                         /* state size: 16 */
    int R;                         /* dt_rank, 1 .. 64 */
    int d_conv;                    /* odd, 1 .. 7 */
    const void *x;                 /* (B, H, W, d_model) bf16 */
    const void *in_proj_weight;    /* (2D, d_model) bf16 */
    const float *in_proj_bias;     /* (2D) fp32, or NULL for none */
    const float *conv_weight;      /* (D, d_conv, d_conv) fp32 */
    const float *conv_bias;        /* (D) fp32, or NULL for none */
    const void *x_proj_weight;     /* (4, R+2N, D) bf16 */
    const float *dt_projs_weight;  /* (4, D, R) fp32 */
    const float *dt_projs_bias;    /* (4*D) fp32, or NULL for zero */
    const float *A_logs;           /* (4*D, N) fp32 */
    const float *Ds;               /* (4*D) fp32, or NULL for zero */
    const float *out_norm_weight;  /* (D) fp32 */
    const float *out_norm_bias;    /* (D) fp32 */
    float out_norm_eps;            /* > 0; LayerNorm's default is 1e-5 */
    const void *out_proj_weight;   /* (d_model, D) bf16 */
    const float *out_proj_bias;    /* (d_model) fp32, or NULL for none */
    void *out;                     /* (B, H, W, d_model) of type out_dtype; must not alias an
                                      input */
    int out_dtype;                 /* SS2D_F32 or SS2D_BF16 */
} ss2d_block_args;

/* Bytes of device workspace ss2d_block_forward needs (xz, x_c, y, g and the core's own
 * workspace), or (size_t)-1 if the arguments are invalid.  out is not read. */
size_t ss2d_block_forward_workspace(const ss2d_block_args *args);

/* The SS2D block's forward pass as described above.  Enqueues five steps on `stream`
 * (the input projection, the convolution, the core's launches, the normalisation with the
 * gate, the output projection) and returns; no allocation, no synchronisation.
 *   workspace : at least ss2d_block_forward_workspace(args) bytes, 16-byte aligned, not
 *               overlapping out; contents need not be initialised and are overwritten.
 * Every tensor pointer must be 16-byte aligned (else SS2D_ERR_MISALIGNED).  Shapes outside
 * the limits above, or that the core's projection form rejects, return
 * SS2D_ERR_UNSUPPORTED and enqueue nothing.  The tensor-core kernels' bounded waits set an
 * error word that ss2d_block_device_status reads. */
int ss2d_block_forward(const ss2d_block_args *args, void *workspace, size_t workspace_bytes, void *stream);

/* Device-side status of the last ss2d_block_forward on this workspace: SS2D_OK, or
 * SS2D_ERR_DEVICE if a bounded wait of one of its tensor-core kernels (the two
 * projections, the core's x_proj GEMM) ran out, in which case out is not valid.
 * Synchronises `stream`. */
int ss2d_block_device_status(const ss2d_block_args *args, const void *workspace, void *stream);

/* Diagnostic (no counterpart in the SS2D pages): runs the error path of the tensor-core
 * kernels' bounded waits on purpose.  One CTA allocates tensor memory, waits on an mbarrier
 * that nothing arrives at for spin_limit polls (1 .. 2^20; a poll takes about 4 us on the
 * B200, and the library's own waits give up after 2^19 polls), then does what the GEMM kernels do
 * when a wait runs out: sets *error_word to 1, frees its tensor memory and returns.  Point
 * error_word at the error word of a projection-form workspace (its first 4 bytes) to see
 * ss2d_device_status report SS2D_ERR_DEVICE from a context that stays usable.  Enqueued on
 * `stream`; returns SS2D_ERR_INVALID_ARG for a NULL word or a limit out of range. */
int ss2d_diag_bounded_wait(int *error_word, long long spin_limit, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SS2D_H */
