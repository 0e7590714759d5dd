// Host side of libct.so: descriptor validation, the output-size / padding
// resolver, the stride-phase table, kernel choice and the C entry points.
//
// Sources: ai.onnx.ConvTranspose README ("Inputs", "Outputs", "Attributes",
// "Type constraints"); ClikaRT::ops::conv_transpose (layout paragraph and
// "Throws").
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <new>

#include "ct_internal.h"

using namespace ct;

namespace {

// Split a total padding into (begin, end) with the odd unit, sign included,
// at the end (odd_at_end) or at the beginning.  C++ division truncates toward
// zero, which keeps that placement for negative totals too.
void split_total(int64_t total, bool odd_at_end, int64_t *pb, int64_t *pe) {
    const int64_t half = total / 2;
    const int64_t extra = total - 2 * half;
    if (odd_at_end) {
        *pb = half;
        *pe = half + extra;
    } else {
        *pb = half + extra;
        *pe = half;
    }
}

// Size limits that keep every product below in int64: a batch, channel,
// group, spatial size, kernel size, stride, dilation, pad or requested output
// size at most 2^30 in magnitude, and at most 2^60 elements in X, W or Y.
constexpr int64_t kMaxDim = int64_t(1) << 30;
constexpr int64_t kMaxElems = int64_t(1) << 60;

// a * b when both are in [0, kMaxElems] and so is the product, else -1
int64_t mul_capped(int64_t a, int64_t b) {
    if (a < 0 || b < 0) return -1;
    if (a != 0 && b > kMaxElems / a) return -1;
    return a * b;
}

// Validate and resolve a descriptor into a plan's geometry.
ct_status resolve(const ct_desc *d, Plan *p) {
    if (!d) return CT_ERR_NULL;
    if (d->rank < 1 || d->rank > 3) return CT_ERR_SPAN;
    if (d->dtype != CT_F32 && d->dtype != CT_F16) return CT_ERR_DTYPE;
    if (d->layout != CT_NCHW && d->layout != CT_NHWC) return CT_ERR_DTYPE;
    if (d->auto_pad < CT_AUTOPAD_NOTSET || d->auto_pad > CT_AUTOPAD_VALID) return CT_ERR_ATTR;
    if (d->algo < CT_ALGO_AUTO || d->algo > CT_ALGO_DENSE_TC_PAIR) return CT_ERR_ATTR;
    if (d->activation != CT_ACT_IDENTITY && d->activation != CT_ACT_RELU) return CT_ERR_ATTR;
    const int r = d->rank;
    if (d->N < 0 || d->C < 0 || d->N > kMaxDim || d->C > kMaxDim) return CT_ERR_ATTR;
    if (d->group <= 0 || d->C % d->group != 0) return CT_ERR_CHANNELS;
    if (d->w_dims[0] != d->C) return CT_ERR_CHANNELS;
    const int64_t mg = d->layout == CT_NCHW ? d->w_dims[1] : d->w_dims[r + 1];
    if (mg <= 0) return CT_ERR_CHANNELS;
    if (mg > kMaxDim || d->group > kMaxDim) return CT_ERR_ATTR;
    const int64_t M = mg * d->group;
    if (d->bias_len < 0 || (d->bias_len != 0 && d->bias_len != M)) return CT_ERR_CHANNELS;

    p->desc = *d;
    p->rank = r;
    p->dtype = d->dtype;
    p->layout = d->layout;
    p->N = d->N;
    p->C = d->C;
    p->M = M;
    p->G = d->group;
    p->Cg = d->C / d->group;
    p->Mg = mg;
    p->has_bias = d->bias_len != 0;
    p->act = d->activation;

    int64_t in[3], k[3], s[3], dl[3], op[3], natural[3];
    for (int a = 0; a < r; ++a) {
        in[a] = d->in[a];
        k[a] = d->layout == CT_NCHW ? d->w_dims[2 + a] : d->w_dims[1 + a];
        s[a] = d->strides[a];
        dl[a] = d->dilations[a];
        op[a] = d->output_padding[a];
        if (s[a] <= 0 || dl[a] <= 0 || k[a] <= 0 || in[a] < 0) return CT_ERR_ATTR;
        if (s[a] > kMaxDim || dl[a] > kMaxDim || k[a] > kMaxDim || in[a] > kMaxDim) return CT_ERR_ATTR;
        if (!d->has_output_shape &&   // with output_shape the pads are ignored
            (d->pads[a] < -kMaxDim || d->pads[a] > kMaxDim || d->pads[r + a] < -kMaxDim ||
             d->pads[r + a] > kMaxDim))
            return CT_ERR_ATTR;
        if (d->has_output_shape && (d->output_shape[a] < -kMaxDim || d->output_shape[a] > kMaxDim))
            return CT_ERR_ATTR;
        const int64_t lim = s[a] > dl[a] ? s[a] : dl[a];
        if (op[a] < 0 || op[a] >= lim) return CT_ERR_ATTR;
        if (d->has_kernel_shape && d->kernel_shape[a] != k[a]) return CT_ERR_ATTR;
        natural[a] = s[a] * (in[a] - 1) + op[a] + (k[a] - 1) * dl[a] + 1;
    }
    if (d->auto_pad != CT_AUTOPAD_NOTSET) {
        for (int a = 0; a < 2 * r; ++a)
            if (d->pads[a] != 0) return CT_ERR_ATTR;
    }
    int64_t pb[3], pe[3], out[3];
    for (int a = 0; a < r; ++a) {
        if (d->has_output_shape) {
            if (d->auto_pad == CT_AUTOPAD_VALID) {
                if (d->output_shape[a] != natural[a]) return CT_ERR_ATTR;
                pb[a] = pe[a] = 0;
            } else {
                split_total(natural[a] - d->output_shape[a],
                            d->auto_pad != CT_AUTOPAD_SAME_LOWER, &pb[a], &pe[a]);
            }
        } else if (d->auto_pad == CT_AUTOPAD_NOTSET) {
            pb[a] = d->pads[a];
            pe[a] = d->pads[r + a];
        } else if (d->auto_pad == CT_AUTOPAD_VALID) {
            pb[a] = pe[a] = 0;
        } else {
            split_total(natural[a] - in[a] * s[a], d->auto_pad == CT_AUTOPAD_SAME_UPPER,
                        &pb[a], &pe[a]);
        }
        out[a] = natural[a] - pb[a] - pe[a];
        if (out[a] <= 0) return CT_ERR_ATTR;
    }
    // element counts of X, W and Y
    int64_t nx = mul_capped(d->N, d->C), nw = mul_capped(d->C, mg), ny = mul_capped(d->N, M);
    for (int a = 0; a < r; ++a) {
        nx = mul_capped(nx, in[a]);
        nw = mul_capped(nw, k[a]);
        ny = mul_capped(ny, out[a]);
    }
    if (nx < 0 || nw < 0 || ny < 0) return CT_ERR_ATTR;
    // pad to three axes, the given ones innermost
    for (int a = 0; a < 3; ++a) {
        const int src = a - (3 - r);
        if (src < 0) {
            p->in[a] = 1; p->k[a] = 1; p->s[a] = 1; p->d[a] = 1;
            p->pb[a] = 0; p->pe[a] = 0; p->op[a] = 0; p->out[a] = 1;
        } else {
            p->in[a] = in[src]; p->k[a] = k[src]; p->s[a] = s[src]; p->d[a] = dl[src];
            p->pb[a] = pb[src]; p->pe[a] = pe[src]; p->op[a] = op[src]; p->out[a] = out[src];
        }
    }
    return CT_OK;
}

// Per axis and output phase r: the taps landing on o = s*J + r and the
// number of such outputs.  Tabled only for strides up to 64.
void build_phase_table(Plan *p) {
    p->tabled = true;
    for (int a = 0; a < 3; ++a)
        if (p->s[a] > 64) p->tabled = false;
    if (!p->tabled) return;
    for (int a = 0; a < 3; ++a) {
        for (int64_t r = 0; r < p->s[a]; ++r) {
            std::vector<Tap> &t = p->taps[a][r];
            t.clear();
            // tap order: increasing input offset e, i.e. decreasing k (the
            // phase's taps reversed)
            for (int64_t k = p->k[a] - 1; k >= 0; --k) {
                const int64_t num = r + p->pb[a] - k * p->d[a];
                int64_t m = num % p->s[a];
                if (m != 0) continue;
                t.push_back(Tap{(int32_t)k, (int32_t)(num / p->s[a])});
            }
            p->nJ[a][r] = p->out[a] > r ? ceil_div(p->out[a] - r, p->s[a]) : 0;
        }
    }
}

void choose(Plan *p) {
    const int want = p->desc.algo;
    p->algo = CT_ALGO_GENERIC;
    if (want == CT_ALGO_GENERIC) return;
    // tiny problems: one gather launch beats any tiled kernel's set-up
    const double flop = 2.0 * p->N * p->C * p->Mg * numel_in(*p) * numel_k(*p);
    if (want == CT_ALGO_AUTO && flop < 1e7) return;
    if (((want == CT_ALGO_AUTO && dense_pair_preferred(*p)) || want == CT_ALGO_DENSE_TC_PAIR) &&
        dense_pair_supports(*p)) {
        p->algo = CT_ALGO_DENSE_TC_PAIR;
    } else if (want == CT_ALGO_DENSE_TC_PAIR) {
        p->algo = -1;
    } else if ((want == CT_ALGO_AUTO || want == CT_ALGO_DENSE_TC) && dense_tc_supports(*p)) {
        p->algo = CT_ALGO_DENSE_TC;
    } else if ((want == CT_ALGO_AUTO || want == CT_ALGO_DENSE_TC || want == CT_ALGO_DENSE_TC_PERTAP) &&
               dense_pertap_supports(*p)) {
        p->algo = CT_ALGO_DENSE_TC_PERTAP;
    } else if ((want == CT_ALGO_AUTO || want == CT_ALGO_GROUPED) && grouped_supports(*p)) {
        p->algo = CT_ALGO_GROUPED;
    } else if ((want == CT_ALGO_AUTO || want == CT_ALGO_FP32_GEMM) && fp32_gemm_supports(*p)) {
        p->algo = CT_ALGO_FP32_GEMM;
    } else if (want == CT_ALGO_AUTO && dense_pair_supports(*p)) {
        // dense shapes the tuned choices above do not take (more than 256
        // output channels, for one)
        p->algo = CT_ALGO_DENSE_TC_PAIR;
    } else if (want != CT_ALGO_AUTO) {
        p->algo = -1;
    }
}

// sm_100 check of the current device, cached per device ordinal.
std::atomic<int> g_dev_ok[64];

ct_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return CT_ERR_DEVICE;
    }
    if (dev < 0 || dev >= 64) return CT_ERR_DEVICE;
    int v = g_dev_ok[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            cudaGetLastError();
            return CT_ERR_DEVICE;
        }
        v = major == 10 ? 1 : 2;
        g_dev_ok[dev].store(v, std::memory_order_relaxed);
    }
    return v == 1 ? CT_OK : CT_ERR_DEVICE;
}

bool aligned(const void *ptr, size_t a) { return ((uintptr_t)ptr % a) == 0; }

}  // namespace

extern "C" {

ct_status ct_output_shape(const ct_desc *desc, int64_t y_dims[5], int64_t pad_begin[3],
                          int64_t pad_end[3]) {
    if (!desc || !y_dims) return CT_ERR_NULL;
    Plan *p = new (std::nothrow) Plan();
    if (!p) return CT_ERR_NOMEM;
    ct_status st = resolve(desc, p);
    if (st == CT_OK) {
        const int r = p->rank;
        y_dims[0] = p->N;
        if (p->layout == CT_NCHW) {
            y_dims[1] = p->M;
            for (int a = 0; a < r; ++a) y_dims[2 + a] = p->out[3 - r + a];
        } else {
            for (int a = 0; a < r; ++a) y_dims[1 + a] = p->out[3 - r + a];
            y_dims[1 + r] = p->M;
        }
        for (int a = r + 2; a < 5; ++a) y_dims[a] = 0;
        for (int a = 0; a < 3; ++a) {
            if (pad_begin) pad_begin[a] = a < r ? p->pb[3 - r + a] : 0;
            if (pad_end) pad_end[a] = a < r ? p->pe[3 - r + a] : 0;
        }
    }
    delete p;
    return st;
}

ct_status ct_plan(const ct_desc *desc, ct_plan_t **out) {
    if (!desc || !out) return CT_ERR_NULL;
    *out = nullptr;
    Plan *p = new (std::nothrow) Plan();
    if (!p) return CT_ERR_NOMEM;
    ct_status st = resolve(desc, p);
    if (st != CT_OK) {
        delete p;
        return st;
    }
    build_phase_table(p);
    choose(p);
    if (p->algo < 0) {
        delete p;
        return CT_ERR_UNSUPPORTED;
    }
    p->ws_bytes = 0;
    p->launches = 1;
    switch (p->algo) {
        case CT_ALGO_DENSE_TC:
            dense_tc_setup(*p);
            p->packed_bytes = dense_tc_packed_bytes(*p);
            p->ws_bytes = dense_tc_ws_bytes(*p);
            break;
        case CT_ALGO_DENSE_TC_PAIR:
            dense_pair_setup(*p);
            p->packed_bytes = dense_pair_packed_bytes(*p);
            p->ws_bytes = dense_pair_ws_bytes(*p);
            break;
        case CT_ALGO_DENSE_TC_PERTAP:
            dense_pertap_setup(*p);
            p->packed_bytes = dense_pertap_packed_bytes(*p);
            p->ws_bytes = dense_pertap_ws_bytes(*p);
            break;
        case CT_ALGO_GROUPED:
            grouped_plan(*p);
            p->packed_bytes = grouped_packed_bytes(*p);
            break;
        case CT_ALGO_FP32_GEMM:
            fp32_gemm_plan(*p);
            p->packed_bytes = fp32_gemm_packed_bytes(*p);
            break;
        default: p->packed_bytes = generic_packed_bytes(*p); break;
    }
    *out = reinterpret_cast<ct_plan_t *>(p);
    return CT_OK;
}

const char *ct_plan_kernel(const ct_plan_t *plan) {
    if (!plan) return "";
    switch (reinterpret_cast<const Plan *>(plan)->algo) {
        case CT_ALGO_DENSE_TC: return "dense_tc";
        case CT_ALGO_DENSE_TC_PERTAP: return "dense_tc_pertap";
        case CT_ALGO_DENSE_TC_PAIR: return "dense_tc_pair";
        case CT_ALGO_FP32_GEMM: return "fp32_gemm";
        case CT_ALGO_GROUPED: return "grouped";
        default: return "generic";
    }
}

ct_status ct_plan_launches(const ct_plan_t *plan, int32_t *launches) {
    if (!plan || !launches) return CT_ERR_NULL;
    const Plan &p = *reinterpret_cast<const Plan *>(plan);
    *launches = p.N * p.M * numel_out(p) == 0 ? 0 : p.launches;
    return CT_OK;
}

ct_status ct_prepacked_weight_bytes(const ct_plan_t *plan, size_t *bytes) {
    if (!plan || !bytes) return CT_ERR_NULL;
    *bytes = reinterpret_cast<const Plan *>(plan)->packed_bytes;
    return CT_OK;
}

ct_status ct_workspace_bytes(const ct_plan_t *plan, size_t *bytes) {
    if (!plan || !bytes) return CT_ERR_NULL;
    *bytes = reinterpret_cast<const Plan *>(plan)->ws_bytes;
    return CT_OK;
}

ct_status ct_prepack_weights(const ct_plan_t *plan, const void *w, void *w_packed, void *stream) {
    if (!plan || !w_packed) return CT_ERR_NULL;
    const Plan &p = *reinterpret_cast<const Plan *>(plan);
    if (!w && p.C * p.Mg * numel_k(p) > 0) return CT_ERR_NULL;
    if (!aligned(w_packed, 16)) return CT_ERR_ALIGN;
    ct_status st = check_device();
    if (st != CT_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (p.algo) {
        case CT_ALGO_DENSE_TC: return dense_tc_prepack(p, w, w_packed, s);
        case CT_ALGO_DENSE_TC_PERTAP: return dense_pertap_prepack(p, w, w_packed, s);
        case CT_ALGO_DENSE_TC_PAIR: return dense_pair_prepack(p, w, w_packed, s);
        case CT_ALGO_GROUPED: return grouped_prepack(p, w, w_packed, s);
        case CT_ALGO_FP32_GEMM: return fp32_gemm_prepack(p, w, w_packed, s);
        default: return generic_prepack(p, w, w_packed, s);
    }
}

ct_status ct_run(const ct_plan_t *plan, const void *x, const void *w_packed, const void *bias,
                 void *y, void *workspace, void *stream) {
    return ct_run_parts(plan, x, w_packed, bias, y, workspace, stream, CT_PART_ALL);
}

ct_status ct_run_parts(const ct_plan_t *plan, const void *x, const void *w_packed, const void *bias,
                       void *y, void *workspace, void *stream, int32_t parts) {
    if (!plan) return CT_ERR_NULL;
    if (parts & ~CT_PART_ALL) return CT_ERR_ATTR;
    if (parts == 0) return CT_OK;
    const Plan &p = *reinterpret_cast<const Plan *>(plan);
    const int64_t ny = p.N * p.M * numel_out(p);
    if (ny == 0) return CT_OK;   // empty output: nothing to write
    if (!y) return CT_ERR_NULL;
    const bool has_terms = p.N * p.C * numel_in(p) > 0;
    if (has_terms && (!x || !w_packed)) return CT_ERR_NULL;
    if (p.has_bias && !bias) return CT_ERR_NULL;
    if (p.ws_bytes > 0 && !workspace) return CT_ERR_WORKSPACE;
    const size_t eb = elem_bytes(p);
    if (!aligned(y, eb) || (x && !aligned(x, eb)) || (bias && !aligned(bias, eb)))
        return CT_ERR_ALIGN;
    if (p.algo != CT_ALGO_GENERIC) {
        if (!aligned(y, 16) || (x && !aligned(x, 16)) || !aligned(w_packed, 16) ||
            (workspace && !aligned(workspace, 256)))
            return CT_ERR_ALIGN;
    }
    ct_status st = check_device();
    if (st != CT_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (p.algo) {
        case CT_ALGO_DENSE_TC: return dense_tc_run(p, x, w_packed, bias, y, workspace, s, parts);
        case CT_ALGO_DENSE_TC_PERTAP: return dense_pertap_run(p, x, w_packed, bias, y, workspace, s, parts);
        case CT_ALGO_DENSE_TC_PAIR: return dense_pair_run(p, x, w_packed, bias, y, workspace, s, parts);
        case CT_ALGO_FP32_GEMM: return fp32_gemm_run(p, x, w_packed, bias, y, s, parts);
        // one launch: the whole call is its main kernel
        case CT_ALGO_GROUPED: return (parts & CT_PART_MAIN) ? grouped_run(p, x, w_packed, bias, y, s) : CT_OK;
        default: return (parts & CT_PART_MAIN) ? generic_run(p, x, w_packed, bias, y, s) : CT_OK;
    }
}

ct_status ct_take_device_error(void *stream, int32_t *code) {
    if (!code) return CT_ERR_NULL;
    *code = 0;
    ct_status st = check_device();
    if (st != CT_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // module numbers 1..5: dense_tc, dense_tc_pair, dense_tc_pertap, grouped, the self-test
    const int words[5] = {dense_tc_take_error(s), dense_pair_take_error(s), dense_pertap_take_error(s),
                          grouped_take_error(s), selftest_take_error(s)};
    bool cuda_failed = false;
    for (int i = 0; i < 5; ++i) {
        if (words[i] < 0) cuda_failed = true;
        if (words[i] > 0 && *code == 0) *code = (i + 1) * 100 + words[i];
    }
    return (cuda_failed || *code != 0) ? CT_ERR_DEVICE : CT_OK;
}

void ct_plan_destroy(ct_plan_t *plan) { delete reinterpret_cast<Plan *>(plan); }

const char *ct_status_string(ct_status status) {
    switch (status) {
        case CT_OK: return "ok";
        case CT_ERR_CHANNELS: return "channel/group arithmetic inconsistent (C, group, W dims or bias length)";
        case CT_ERR_SPAN: return "span length inconsistent (rank or attribute length)";
        case CT_ERR_DTYPE: return "dtype or layout not served";
        case CT_ERR_ATTR: return "attribute invalid (stride, dilation, kernel, pads, output_padding, output_shape, activation)";
        case CT_ERR_ALIGN: return "device pointer misaligned for the chosen kernel";
        case CT_ERR_NULL: return "required pointer is NULL";
        case CT_ERR_DEVICE: return "CUDA device error (not sm_100, or launch failure)";
        case CT_ERR_WORKSPACE: return "workspace missing";
        case CT_ERR_UNSUPPORTED: return "forced algorithm cannot serve this shape";
        case CT_ERR_NOMEM: return "host allocation failed";
    }
    return "unknown status";
}

}  // extern "C"
