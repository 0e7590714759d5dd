/*
 * ct.h -- C ABI of the B200 (sm_100a) ONNX ConvTranspose library (libct.so).
 *
 * The operation (ai.onnx.ConvTranspose README, "Description", "Inputs",
 * "Outputs", "Attributes" and "Type constraints"): Y is the transposed
 * (fractionally strided) convolution of X with W, plus an optional bias B
 * per output channel.  With pad_begin/pad_end resolved per spatial axis a,
 * input position i and kernel tap k land on output position
 *
 *     o_a = i_a * strides_a - pad_begin_a + k_a * dilations_a
 *
 * and Y[n, g*M/group + m, o] is the sum of X[n, g*C/group + c, i] *
 * W[g*C/group + c, m, k] over every (c, i, k) landing on o, plus B[...].
 * The output size per axis is
 *
 *     out_a = strides_a*(in_a - 1) + output_padding_a + (k_a - 1)*dilations_a
 *             + 1 - pad_begin_a - pad_end_a.
 *
 * Two layouts are served:
 *   CT_NCHW  channels-first, as the ai.onnx.ConvTranspose README states it:
 *            X[N, C, D1..Dr], W[C, M/group, k1..kr], Y[N, M, out1..outr].
 *   CT_NHWC  channels-last, as ClikaRT::ops::conv_transpose states it (its
 *            layout paragraph): X[N, D1..Dr, C], W[C, k1..kr, M/group]
 *            (input-channel first), Y[N, out1..outr, M].
 * X, W, B and Y share one element type T in {float32, float16} (README,
 * "Type constraints").  All tensors are dense, row-major, in device memory.
 *
 * Ownership: the caller owns every device buffer and the stream; the library
 * owns only the opaque plan.  No entry point calls a device allocator; the
 * device memory libct.so holds by itself is its code and its file-scope
 * device arrays (the ct_run_noalloc workspace among them), which CUDA loads
 * onto a device with the library's kernels, at the latest on the first call
 * that uses that device.
 * Errors: every entry point returns a ct_status; nothing is thrown across the
 * ABI, nothing is printed.  Validation happens in ct_plan, before any launch.
 * The status classes mirror the error classes of ClikaRT::ops::conv_transpose
 * ("Throws": channel/group arithmetic, span lengths, dtype).
 */
#ifndef CT_H_
#define CT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CT_API __attribute__((visibility("default")))
#else
#define CT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ct_status {
    CT_OK = 0,
    CT_ERR_CHANNELS = 1,   /* C % group != 0, W dims inconsistent with C/group, or bias length != M */
    CT_ERR_SPAN = 2,       /* rank outside 1..3, or an attribute span of the wrong length */
    CT_ERR_DTYPE = 3,      /* element type not float32/float16, or layout unknown */
    CT_ERR_ATTR = 4,       /* stride/dilation/kernel <= 0, output_padding >= max(stride, dilation),
                              kernel_shape != W dims, pads with auto_pad, empty or inconsistent output */
    CT_ERR_ALIGN = 5,      /* a device pointer is not aligned as the chosen kernel requires */
    CT_ERR_NULL = 6,       /* a required pointer is NULL */
    CT_ERR_DEVICE = 7,     /* the current device is not sm_100, or a CUDA launch failed */
    CT_ERR_WORKSPACE = 8,  /* workspace pointer missing although ct_workspace_bytes > 0 */
    CT_ERR_UNSUPPORTED = 9,/* a forced algorithm cannot serve this shape */
    CT_ERR_NOMEM = 10      /* host allocation of the plan failed */
} ct_status;

typedef enum ct_dtype { CT_F32 = 0, CT_F16 = 1 } ct_dtype;
typedef enum ct_layout { CT_NCHW = 0, CT_NHWC = 1 } ct_layout;

/* auto_pad (README "Attributes"): NOTSET uses pads; SAME_UPPER/SAME_LOWER give
 * out = in * stride with the odd unit of the total padding at the end / the
 * beginning; VALID pads nothing. */
typedef enum ct_autopad {
    CT_AUTOPAD_NOTSET = 0,
    CT_AUTOPAD_SAME_UPPER = 1,
    CT_AUTOPAD_SAME_LOWER = 2,
    CT_AUTOPAD_VALID = 3
} ct_autopad;

/* Kernel selection: CT_ALGO_AUTO lets ct_plan choose; the others force one
 * kernel (for tests) and make ct_plan return CT_ERR_UNSUPPORTED when that
 * kernel cannot serve the shape. */
typedef enum ct_algo {
    CT_ALGO_AUTO = 0,
    CT_ALGO_GENERIC = 1,   /* per-output gather, any shape */
    CT_ALGO_DENSE_TC = 2,  /* fp16 group-1 phase GEMM on tcgen05 tensor cores */
    CT_ALGO_FP32_GEMM = 3, /* fp32 group-1 register-tiled FFMA phase GEMM */
    CT_ALGO_GROUPED = 4,   /* fp16 grouped phase kernel (mma.sync), small per-group slabs */
    CT_ALGO_DENSE_TC_PERTAP = 5, /* fp16 group-1 tcgen05 phase GEMM, one input load per tap
                                    (the general fallback of CT_ALGO_DENSE_TC) */
    CT_ALGO_DENSE_TC_PAIR = 6    /* group-1 phase GEMM, each MMA spanning the two SMs of a CTA
                                    pair (tcgen05 cta_group::2), either layout; fp16 (chosen
                                    automatically for channels-first with one or two spatial
                                    axes) or fp32 as 3xTF32 (TF32 high part and remainder of
                                    both operands, three MMAs per step; chosen automatically
                                    for fp32).  The workspace holds a zero-padded
                                    channels-last copy of X (two planes, high parts and
                                    remainders, for fp32) */
} ct_algo;

/* Activation applied to every output after the bias (ClikaRT::ops::
 * conv_transpose, parameter `activation`, default Identity).  The page does
 * not list the Activation members; this library offers identity and ReLU
 * (max(v, 0)), applied in fp32 before the output is rounded to its dtype.
 * Any other value is CT_ERR_ATTR. */
typedef enum ct_activation {
    CT_ACT_IDENTITY = 0,
    CT_ACT_RELU = 1
} ct_activation;

/* One ConvTranspose call.  Every array has 3 slots; only the first `rank`
 * (and 2*rank for pads) are read. */
typedef struct ct_desc {
    int32_t rank;              /* spatial rank r, 1..3 */
    int32_t dtype;             /* ct_dtype */
    int32_t layout;            /* ct_layout */
    int32_t auto_pad;          /* ct_autopad */
    int64_t N;                 /* batch */
    int64_t C;                 /* input channels */
    int64_t in[3];             /* input spatial sizes D1..Dr */
    int64_t w_dims[5];         /* W's dims as declared: CT_NCHW [C, M/group, k1..kr],
                                  CT_NHWC [C, k1..kr, M/group] */
    int64_t group;
    int64_t bias_len;          /* 0: no bias; else must equal M */
    int64_t strides[3];
    int64_t dilations[3];
    int64_t pads[6];           /* README order: begins of every axis, then ends */
    int64_t output_padding[3];
    int32_t has_kernel_shape;
    int32_t has_output_shape;
    int64_t kernel_shape[3];
    int64_t output_shape[3];
    int32_t algo;              /* ct_algo */
    int32_t activation;        /* ct_activation */
} ct_desc;

typedef struct ct_plan_s ct_plan_t;

/* Resolve the output: Y's dims in the descriptor's layout (rank + 2 entries)
 * and the begin/end pads per axis.  Pure host code, no device touched.
 * Implements the output-size rule above with the auto_pad / output_shape /
 * output_padding rows of the README's "Attributes" table.  Library limits
 * (CT_ERR_ATTR beyond them, so that no size arithmetic overflows int64):
 * N, C, M/group, group, every spatial size, kernel size, stride, dilation,
 * pad and requested output size at most 2^30 in magnitude; X, W and Y each
 * at most 2^60 elements. */
CT_API ct_status ct_output_shape(const ct_desc *desc, int64_t y_dims[5],
                          int64_t pad_begin[3], int64_t pad_end[3]);

/* Validate the descriptor, resolve it, build the stride-phase table and
 * choose a kernel.  Pure host code.  On success *out owns a plan that the
 * caller frees with ct_plan_destroy. */
CT_API ct_status ct_plan(const ct_desc *desc, ct_plan_t **out);

/* Name of the kernel the plan runs ("generic", "dense_tc", ...).  The string
 * is static; NULL plan gives "". */
CT_API const char *ct_plan_kernel(const ct_plan_t *plan);

/* Number of kernels one ct_run of this plan launches (for launch accounting). */
CT_API ct_status ct_plan_launches(const ct_plan_t *plan, int32_t *launches);

/* Bytes of device memory the caller provides for the pre-packed weight. */
CT_API ct_status ct_prepacked_weight_bytes(const ct_plan_t *plan, size_t *bytes);

/* Bytes of device scratch ct_run needs (0 when the kernel needs none). */
CT_API ct_status ct_workspace_bytes(const ct_plan_t *plan, size_t *bytes);

/* Re-lay W (the declared layout, device memory) into the plan's packed form
 * in w_packed (ct_prepacked_weight_bytes bytes, 16-byte aligned): taps split
 * into stride phases, tap order reversed within a phase, the reduction axis
 * contiguous (ai.onnx.ConvTranspose README, "Files": the 2-D/3-D weight
 * reorder templates).  Asynchronous on `stream` (a cudaStream_t, NULL for the
 * legacy default stream). */
CT_API ct_status ct_prepack_weights(const ct_plan_t *plan, const void *w, void *w_packed,
                             void *stream);

/* Y = ConvTranspose(X, W, B).  x, w_packed, bias (NULL when bias_len == 0),
 * y and workspace are device pointers; y is fully overwritten, including
 * positions no tap reaches, which receive the bias (or zero).  Asynchronous
 * on `stream`; a launch error returns CT_ERR_DEVICE. */
CT_API ct_status ct_run(const ct_plan_t *plan, const void *x, const void *w_packed,
                 const void *bias, void *y, void *workspace, void *stream);

/* Parts of one ct_run, for measuring them apart (ct_run_parts).  A call
 * consists of preparation launches (the re-layout of X into the workspace,
 * and the bias fill of outputs no tap reaches) followed by one main kernel
 * (the phase GEMM or gather).  Plans whose call is a single kernel have no
 * preparation: CT_PART_PREPARE alone launches nothing for them. */
#define CT_PART_PREPARE 1
#define CT_PART_MAIN 2
#define CT_PART_ALL 3

/* ct_run restricted to the parts in `parts` (a mask of CT_PART_*; 0 does
 * nothing, other bits are CT_ERR_ATTR).  ct_run(...) is ct_run_parts(...,
 * CT_PART_ALL).  CT_PART_MAIN alone reads the workspace and Y as an earlier
 * CT_PART_PREPARE call with the same x, workspace and y left them: a
 * benchmark prepares once and then times the main kernel by itself.  With
 * anything else in the workspace the main kernel still reads and writes
 * only inside the planned buffers, but Y is not the operator's result.
 * Arguments, alignment and errors as for ct_run. */
CT_API ct_status ct_run_parts(const ct_plan_t *plan, const void *x, const void *w_packed,
                              const void *bias, void *y, void *workspace, void *stream,
                              int32_t parts);

/* Size of the device array that ct_run_noalloc uses as its workspace.  Every
 * GPU that loads libct.so holds this much device memory until the process
 * exits. */
#define CT_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* ct_run for callers that cannot allocate device memory while running, such
 * as a plugin inside an engine that owns all device memory, or a loop whose
 * rules forbid allocation after start-up.  The ONNX page and the ClikaRT page
 * have no counterpart of this call; it exists only for such callers.  The
 * caller still passes x, w_packed, bias and y as for ct_run.  The workspace
 * comes from a fixed array of CT_NOALLOC_SCRATCH_BYTES inside the library:
 * plans whose ct_workspace_bytes exceed that return CT_ERR_WORKSPACE.  Every
 * call looks up the array's device address on the current device
 * (cudaGetSymbolAddress; host code only ever sees a stand-in for the array,
 * never its device address).  With CUDA's lazy module loading the first such
 * lookup on a device loads the module that holds the array, which takes
 * CT_NOALLOC_SCRATCH_BYTES of device memory at that moment: make the first
 * call on each device at start-up, before any stream capture and before the
 * caller hands the rest of the device memory to its own allocator.  Later
 * calls allocate nothing.  All calls share the one array (it keeps the last
 * call's contents; the kernels overwrite all workspace bytes they read), so
 * calls whose GPU work overlaps in time, for example on two streams, race on
 * it and must be serialised by the caller. */
CT_API ct_status ct_run_noalloc(const ct_plan_t *plan, const void *x, const void *w_packed,
                                const void *bias, void *y, void *stream);

CT_API void ct_plan_destroy(ct_plan_t *plan);

/* Static, human-readable text for a status code. */
CT_API const char *ct_status_string(ct_status status);

/* Failure report of the kernels' bounded waits.  Every wait of the
 * tensor-core and grouped kernels on an mbarrier gives up after about one
 * second of SM clock; the kernel then records a code in its module's device
 * error word, skips the rest of its work (so Y is not valid) and returns, and
 * the device stays usable.  This call waits for `stream` (work that ran
 * earlier on other streams must be finished by the caller), then reads and
 * clears the error words of the current device.  *code = 0 and CT_OK when no
 * wait ran out since the last call; otherwise *code = 100 * module + wait
 * site (module 1 dense_tc, 2 dense_tc_pair, 3 dense_tc_pertap, 4 grouped,
 * 5 the self-test below) and CT_ERR_DEVICE.  CT_ERR_DEVICE with *code = 0
 * means a CUDA call failed (or the current device is not an sm_100 part). */
CT_API ct_status ct_take_device_error(void *stream, int32_t *code);

/* Self-test of the bounded-wait failure path (no counterpart on the pages).
 * One block of one thread runs the steps every tensor-core kernel takes when
 * a wait runs out: it starts a bulk copy of 4 KB into its shared memory,
 * then waits, with a limit of `limit_cycles` SM clock cycles (1 .. 2^31),
 * on an mbarrier that nothing ever arrives at.  When the limit runs out it
 * records wait site 1 in module 5's error word, waits (with the kernels'
 * usual one-second limit) for its copy still in flight, and returns.  So
 * after a call, ct_take_device_error reports code 501 and the device stays
 * usable; site 2 would mean the copy never completed.  Asynchronous on
 * `stream`; CT_ERR_ATTR for a limit outside the range. */
CT_API ct_status ct_selftest_wait_timeout(void *stream, int64_t limit_cycles);

#ifdef __cplusplus
}
#endif

#endif /* CT_H_ */
