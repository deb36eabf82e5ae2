// C ABI of the mLSTM library: argument validation and kernel selection.
// Declarations and the contract of every entry point: include/xlstm_mlstm.h.
#include <cmath>
#include <cstring>

#include "common.cuh"

namespace {

using xlstm::FwdArgs;

constexpr size_t kWorkspaceBytes = 256;   // status block (16 B), padded

bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
    const char *lo;
    size_t bytes;
};

bool overlap(Range a, Range b) {
    if (!a.lo || !b.lo || a.bytes == 0 || b.bytes == 0) return false;
    return a.lo < b.lo + b.bytes && b.lo < a.lo + a.bytes;
}

Range rg(const void *p, size_t bytes) { return Range{static_cast<const char *>(p), bytes}; }

bool dims_ok(const xlstm_mlstm_desc_t *d) {
    if (d->B < 1 || d->H < 1 || d->T < 0) return false;
    if (d->d_qk < 16 || d->d_qk > 512 || d->d_qk % 16) return false;
    if (d->d_v < 16 || d->d_v > 512 || d->d_v % 16) return false;
    if (d->qkv_dtype != XLSTM_F32 && d->qkv_dtype != XLSTM_BF16) return false;
    if (!std::isfinite(d->qk_scale)) return false;
    return true;
}

size_t elem(const xlstm_mlstm_desc_t *d) { return d->qkv_dtype == XLSTM_BF16 ? 2 : 4; }

// Chunk lengths each path takes: 64 for every input type; 16, 32 and 128 for fp32
// inputs, which run on the CUDA-core kernel; 128 for bf16 inputs with d_qk <= 128
// on the tensor-core kernel (tensor memory holds the state, its readout copy and
// one chunk's S and H; at d_qk = 256 only L = 64 fits).  Other lengths are
// refused, not rerouted to another kernel.
bool chunk_ok(const xlstm_mlstm_desc_t *d) {
    const int L = d->chunk ? d->chunk : 64;
    if (L == 64) return true;
    if (d->qkv_dtype == XLSTM_F32) return L == 16 || L == 32 || L == 128;
    if (L != 128) return false;
    xlstm::FwdArgs a{};
    a.dtype = d->qkv_dtype; a.chunk = L; a.T = 1; a.dqk = d->d_qk; a.dv = d->d_v;
    return xlstm::chunkwise_tc_shape_ok(a);
}

// Shared validation of the two sequence calls.
// h_elem: bytes per element of h; o (optional input, o_elem bytes per element) is
// the output-gate pre-activation tensor of the chunkwise output stage.
xlstm_status_t check_sequence(const xlstm_mlstm_desc_t *d, const void *q, const void *k,
                              const void *v, const float *ig, const float *fg, const float *C0,
                              const float *n0, const float *m0, const void *h, const float *C1,
                              const float *n1, const float *m1, size_t h_elem = 4,
                              const void *o = nullptr, size_t o_elem = 0) {
    if (!d || !dims_ok(d)) return XLSTM_ERR_INVALID_ARG;
    const int ns = (C0 != nullptr) + (n0 != nullptr) + (m0 != nullptr);
    if (ns != 0 && ns != 3) return XLSTM_ERR_INVALID_ARG;
    if (d->T > 0 && (!q || !k || !v || !ig || !fg || !h)) return XLSTM_ERR_INVALID_ARG;
    const void *all[] = {q, k, v, ig, fg, C0, n0, m0, h, C1, n1, m1, o};
    for (const void *p : all)
        if (!aligned16(p)) return XLSTM_ERR_INVALID_ARG;
    const size_t BH = (size_t)d->B * d->H, T = (size_t)d->T;
    const size_t e = elem(d);
    const Range ins[] = {rg(q, BH * T * d->d_qk * e), rg(k, BH * T * d->d_qk * e),
                         rg(v, BH * T * d->d_v * e), rg(ig, BH * T * 4), rg(fg, BH * T * 4),
                         rg(C0, BH * d->d_v * d->d_qk * 4), rg(n0, BH * d->d_qk * 4), rg(m0, BH * 4),
                         rg(o, BH * T * d->d_v * o_elem)};
    const Range outs[] = {rg(h, BH * T * d->d_v * h_elem), rg(C1, BH * d->d_v * d->d_qk * 4),
                          rg(n1, BH * d->d_qk * 4), rg(m1, BH * 4)};
    for (const Range &o : outs) {
        for (const Range &i : ins)
            if (overlap(o, i)) return XLSTM_ERR_INVALID_ARG;
        for (const Range &o2 : outs)
            if (&o2 != &o && overlap(o, o2)) return XLSTM_ERR_INVALID_ARG;
    }
    return XLSTM_OK;
}

FwdArgs pack(const xlstm_mlstm_desc_t *d, const void *q, const void *k, const void *v,
             const float *ig, const float *fg, const float *C0, const float *n0, const float *m0,
             float *h, float *C1, float *n1, float *m1) {
    FwdArgs a;
    a.B = d->B; a.H = d->H; a.T = d->T; a.dqk = d->d_qk; a.dv = d->d_v;
    a.dtype = d->qkv_dtype; a.scale = d->qk_scale; a.chunk = d->chunk ? d->chunk : 64;
    a.q = q; a.k = k; a.v = v; a.ig = ig; a.fg = fg; a.C0 = C0; a.n0 = n0; a.m0 = m0;
    a.h = h; a.C1 = C1; a.n1 = n1; a.m1 = m1; a.status = nullptr; a.seg_ws = nullptr;
    return a;
}

// T == 0: the final state is the initial one (zero when none was given).
xlstm_status_t pass_state_through(const FwdArgs &a, cudaStream_t s) {
    const size_t BH = (size_t)a.B * a.H;
    const size_t cb = BH * a.dv * a.dqk * 4, nb = BH * a.dqk * 4, mb = BH * 4;
    cudaError_t e = cudaSuccess;
    if (a.C1) e = a.C0 ? cudaMemcpyAsync(a.C1, a.C0, cb, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(a.C1, 0, cb, s);
    if (e == cudaSuccess && a.n1)
        e = a.n0 ? cudaMemcpyAsync(a.n1, a.n0, nb, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(a.n1, 0, nb, s);
    if (e == cudaSuccess && a.m1)
        e = a.m0 ? cudaMemcpyAsync(a.m1, a.m0, mb, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(a.m1, 0, mb, s);
    return e == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t xlstm_mlstm_workspace_size(const xlstm_mlstm_desc_t *desc) {
    return desc ? kWorkspaceBytes : 0;
}

size_t xlstm_mlstm_workspace_size_parallel(const xlstm_mlstm_desc_t *desc) {
    if (!desc) return 0;
    if (!dims_ok(desc)) return kWorkspaceBytes;
    const FwdArgs a = pack(desc, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                           nullptr, nullptr, nullptr);
    const xlstm::SegPlan sp = xlstm::segment_plan(a);
    return kWorkspaceBytes + (sp.nseg > 1 ? sp.bytes : 0);
}

}  // extern "C"

namespace {

// The chunkwise call behind both entry points; a is packed, st the argument check.
xlstm_status_t run_chunkwise(const xlstm_mlstm_desc_t *desc, FwdArgs a, xlstm_status_t st, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
    if (st != XLSTM_OK) return st;
    if (!chunk_ok(desc)) return XLSTM_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < xlstm_mlstm_workspace_size(desc)) return XLSTM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return XLSTM_ERR_INVALID_ARG;
    a.status = static_cast<int32_t *>(workspace);
    if (cudaMemsetAsync(workspace, 0, 16, stream) != cudaSuccess) return XLSTM_ERR_CUDA;
    if (a.T == 0) return pass_state_through(a, stream);
    if (xlstm::chunkwise_tc_supported(a)) {
        // a long sequence with few heads runs in parallel segments when the workspace holds their summaries
        const xlstm::SegPlan sp = xlstm::segment_plan(a);
        if (sp.nseg > 1 && workspace_bytes >= kWorkspaceBytes + sp.bytes)
            a.seg_ws = static_cast<char *>(workspace) + kWorkspaceBytes;
    }
    cudaError_t e = xlstm::chunkwise_tc_supported(a) ? xlstm::launch_chunkwise_tc(a, stream)
                                                     : xlstm::launch_chunkwise_simt(a, stream);
    return e == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}

}  // namespace

extern "C" {

xlstm_status_t xlstm_mlstm_fwd_chunkwise(const xlstm_mlstm_desc_t *desc, const void *q,
                                         const void *k, const void *v, const float *i_pre,
                                         const float *f_pre, const float *C_in, const float *n_in,
                                         const float *m_in, float *h_out, float *C_out,
                                         float *n_out, float *m_out, void *workspace,
                                         size_t workspace_bytes, cudaStream_t stream) {
    const xlstm_status_t st = check_sequence(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, h_out,
                                             C_out, n_out, m_out);
    if (st != XLSTM_OK) return st;
    return run_chunkwise(desc, pack(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, h_out, C_out, n_out, m_out), st,
                         workspace, workspace_bytes, stream);
}

xlstm_status_t xlstm_mlstm_fwd_chunkwise_out(const xlstm_mlstm_desc_t *desc, const xlstm_mlstm_output_t *out,
                                             const void *q, const void *k, const void *v, const float *i_pre,
                                             const float *f_pre, const float *C_in, const float *n_in,
                                             const float *m_in, void *h_out, float *C_out, float *n_out,
                                             float *m_out, void *workspace, size_t workspace_bytes,
                                             cudaStream_t stream) {
    xlstm::OutStage os;
    if (out) {
        const bool ok_o = out->o_pre == nullptr || out->o_dtype == XLSTM_F32 || out->o_dtype == XLSTM_BF16;
        if (!ok_o || (out->h_dtype != XLSTM_F32 && out->h_dtype != XLSTM_BF16)) return XLSTM_ERR_INVALID_ARG;
        os.o = out->o_pre;
        os.o_bf16 = out->o_pre && out->o_dtype == XLSTM_BF16;
        os.h_bf16 = out->h_dtype == XLSTM_BF16;
    }
    const xlstm_status_t st =
        check_sequence(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, h_out, C_out, n_out, m_out,
                       os.h_bf16 ? 2 : 4, os.o, os.o ? (os.o_bf16 ? 2 : 4) : 0);
    if (st != XLSTM_OK) return st;
    FwdArgs a = pack(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, static_cast<float *>(h_out), C_out, n_out,
                     m_out);
    a.out = os;
    return run_chunkwise(desc, a, st, workspace, workspace_bytes, stream);
}

xlstm_status_t xlstm_mlstm_fwd_recurrent(const xlstm_mlstm_desc_t *desc, const void *q,
                                         const void *k, const void *v, const float *i_pre,
                                         const float *f_pre, const float *C_in, const float *n_in,
                                         const float *m_in, float *h_out, float *C_out,
                                         float *n_out, float *m_out, void *workspace,
                                         size_t workspace_bytes, cudaStream_t stream) {
    (void)workspace;
    (void)workspace_bytes;
    xlstm_status_t st = check_sequence(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, h_out,
                                       C_out, n_out, m_out);
    if (st != XLSTM_OK) return st;
    FwdArgs a = pack(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, h_out, C_out, n_out, m_out);
    if (a.T == 0) return pass_state_through(a, stream);
    return xlstm::launch_recurrent(a, stream) == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}

xlstm_status_t xlstm_mlstm_step(const xlstm_mlstm_desc_t *desc, const void *q, const void *k,
                                const void *v, const float *i_pre, const float *f_pre,
                                const float *C, const float *n, const float *m, float *h_out,
                                float *C_new, float *n_new, float *m_new, cudaStream_t stream) {
    if (!desc) return XLSTM_ERR_INVALID_ARG;
    xlstm_mlstm_desc_t d = *desc;
    d.T = 1;
    if (!dims_ok(&d)) return XLSTM_ERR_INVALID_ARG;
    const void *req[] = {q, k, v, i_pre, f_pre, C, n, m, h_out, C_new, n_new, m_new};
    for (const void *p : req)
        if (!p || !aligned16(p)) return XLSTM_ERR_INVALID_ARG;
    const size_t BH = (size_t)d.B * d.H, e = elem(&d);
    const Range ins[] = {rg(q, BH * d.d_qk * e), rg(k, BH * d.d_qk * e), rg(v, BH * d.d_v * e),
                         rg(i_pre, BH * 4), rg(f_pre, BH * 4), rg(C, BH * d.d_v * d.d_qk * 4),
                         rg(n, BH * d.d_qk * 4), rg(m, BH * 4)};
    const Range outs[] = {rg(h_out, BH * d.d_v * 4), rg(C_new, BH * d.d_v * d.d_qk * 4),
                          rg(n_new, BH * d.d_qk * 4), rg(m_new, BH * 4)};
    // An output may coincide exactly with its own state input (in place).
    const int own[] = {-1, 5, 6, 7};
    for (int o = 0; o < 4; ++o) {
        for (int i = 0; i < 8; ++i) {
            if (i == own[o] && outs[o].lo == ins[i].lo) continue;
            if (overlap(outs[o], ins[i])) return XLSTM_ERR_INVALID_ARG;
        }
        for (int o2 = 0; o2 < 4; ++o2)
            if (o2 != o && overlap(outs[o], outs[o2])) return XLSTM_ERR_INVALID_ARG;
    }
    FwdArgs a = pack(&d, q, k, v, i_pre, f_pre, C, n, m, h_out, C_new, n_new, m_new);
    return xlstm::launch_step(a, stream) == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}

xlstm_status_t xlstm_mlstm_segment_summary(const xlstm_mlstm_desc_t *desc, const void *k, const void *v,
                                           const float *i_pre, const float *f_pre, float *C_seg, float *n_seg,
                                           double *F_m, void *workspace, size_t workspace_bytes,
                                           cudaStream_t stream) {
    if (!desc || !dims_ok(desc) || desc->T < 1) return XLSTM_ERR_INVALID_ARG;
    const void *req[] = {k, v, i_pre, f_pre, C_seg, n_seg, F_m};
    for (const void *p : req)
        if (!p || !aligned16(p)) return XLSTM_ERR_INVALID_ARG;
    const size_t BH = (size_t)desc->B * desc->H, T = (size_t)desc->T, e = elem(desc);
    const Range ins[] = {rg(k, BH * T * desc->d_qk * e), rg(v, BH * T * desc->d_v * e), rg(i_pre, BH * T * 4),
                         rg(f_pre, BH * T * 4)};
    const Range outs[] = {rg(C_seg, BH * desc->d_v * desc->d_qk * 4), rg(n_seg, BH * desc->d_qk * 4),
                          rg(F_m, BH * 2 * sizeof(double))};
    for (const Range &o : outs) {
        for (const Range &i : ins)
            if (overlap(o, i)) return XLSTM_ERR_INVALID_ARG;
        for (const Range &o2 : outs)
            if (&o2 != &o && overlap(o, o2)) return XLSTM_ERR_INVALID_ARG;
    }
    FwdArgs a = pack(desc, nullptr, k, v, i_pre, f_pre, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                     nullptr);
    if (!chunk_ok(desc) || !xlstm::summary_supported(a)) return XLSTM_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < kWorkspaceBytes) return XLSTM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return XLSTM_ERR_INVALID_ARG;
    a.status = static_cast<int32_t *>(workspace);
    if (cudaMemsetAsync(workspace, 0, 16, stream) != cudaSuccess) return XLSTM_ERR_CUDA;
    return xlstm::launch_summary(a, C_seg, n_seg, F_m, stream) == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}

xlstm_status_t xlstm_mlstm_combine_states(const xlstm_mlstm_desc_t *desc, int32_t nsum, const float *C_in,
                                          const float *n_in, const float *m_in, const float *C_seg,
                                          const float *n_seg, const double *F_m, float *C_out, float *n_out,
                                          float *m_out, cudaStream_t stream) {
    if (!desc) return XLSTM_ERR_INVALID_ARG;
    xlstm_mlstm_desc_t d = *desc;
    d.T = 1;
    if (!dims_ok(&d) || nsum < 0) return XLSTM_ERR_INVALID_ARG;
    const int ns = (C_in != nullptr) + (n_in != nullptr) + (m_in != nullptr);
    if (ns != 0 && ns != 3) return XLSTM_ERR_INVALID_ARG;
    if (nsum > 0 && (!C_seg || !n_seg || !F_m)) return XLSTM_ERR_INVALID_ARG;
    if (!C_out || !n_out || !m_out) return XLSTM_ERR_INVALID_ARG;
    const void *all[] = {C_in, n_in, m_in, C_seg, n_seg, F_m, C_out, n_out, m_out};
    for (const void *p : all)
        if (!aligned16(p)) return XLSTM_ERR_INVALID_ARG;
    const size_t BH = (size_t)d.B * d.H, S = (size_t)nsum;
    const Range ins[] = {rg(C_in, BH * d.d_v * d.d_qk * 4), rg(n_in, BH * d.d_qk * 4), rg(m_in, BH * 4),
                         rg(C_seg, S * BH * d.d_v * d.d_qk * 4), rg(n_seg, S * BH * d.d_qk * 4),
                         rg(F_m, S * BH * 2 * sizeof(double))};
    const Range outs[] = {rg(C_out, BH * d.d_v * d.d_qk * 4), rg(n_out, BH * d.d_qk * 4), rg(m_out, BH * 4)};
    for (const Range &o : outs) {
        for (const Range &i : ins)
            if (overlap(o, i)) return XLSTM_ERR_INVALID_ARG;
        for (const Range &o2 : outs)
            if (&o2 != &o && overlap(o, o2)) return XLSTM_ERR_INVALID_ARG;
    }
    return xlstm::launch_combine((int)BH, d.d_v, d.d_qk, nsum, C_in, n_in, m_in, C_seg, n_seg, F_m, C_out, n_out,
                                 m_out, stream) == cudaSuccess
               ? XLSTM_OK
               : XLSTM_ERR_CUDA;
}

size_t xlstm_mlstm_bwd_workspace_size(const xlstm_mlstm_desc_t *desc) {
    if (!desc || !dims_ok(desc)) return 0;
    return xlstm::backward_workspace_bytes(desc->B * desc->H, desc->T, desc->d_qk, desc->d_v);
}

xlstm_status_t xlstm_mlstm_bwd_chunkwise(const xlstm_mlstm_desc_t *desc, const void *q, const void *k,
                                         const void *v, const float *i_pre, const float *f_pre,
                                         const float *C_in, const float *n_in, const float *m_in,
                                         const float *dh, const float *dC_out, const float *dn_out, float *dq,
                                         float *dk, float *dv, float *di_pre, float *df_pre, float *dC_in,
                                         float *dn_in, float *dm_in, void *workspace, size_t workspace_bytes,
                                         cudaStream_t stream) {
    if (!desc || !dims_ok(desc)) return XLSTM_ERR_INVALID_ARG;
    const int ns = (C_in != nullptr) + (n_in != nullptr) + (m_in != nullptr);
    if (ns != 0 && ns != 3) return XLSTM_ERR_INVALID_ARG;
    if ((dC_out == nullptr) != (dn_out == nullptr)) return XLSTM_ERR_INVALID_ARG;
    if (desc->T > 0 && (!q || !k || !v || !i_pre || !f_pre || !dh || !dq || !dk || !dv || !di_pre || !df_pre))
        return XLSTM_ERR_INVALID_ARG;
    const void *all[] = {q, k, v, i_pre, f_pre, C_in, n_in, m_in, dh, dC_out, dn_out,
                         dq, dk, dv, di_pre, df_pre, dC_in, dn_in, dm_in};
    for (const void *p : all)
        if (!aligned16(p)) return XLSTM_ERR_INVALID_ARG;
    const size_t BH = (size_t)desc->B * desc->H, T = (size_t)desc->T, e = elem(desc);
    const size_t sC = BH * desc->d_v * desc->d_qk * 4, sn = BH * desc->d_qk * 4, sm = BH * 4;
    const Range ins[] = {rg(q, BH * T * desc->d_qk * e), rg(k, BH * T * desc->d_qk * e), rg(v, BH * T * desc->d_v * e),
                         rg(i_pre, BH * T * 4), rg(f_pre, BH * T * 4), rg(C_in, sC), rg(n_in, sn), rg(m_in, sm),
                         rg(dh, BH * T * desc->d_v * 4), rg(dC_out, sC),
                         rg(dn_out, sn)};
    const Range outs[] = {rg(dq, BH * T * desc->d_qk * 4), rg(dk, BH * T * desc->d_qk * 4),
                          rg(dv, BH * T * desc->d_v * 4), rg(di_pre, BH * T * 4), rg(df_pre, BH * T * 4),
                          rg(dC_in, sC), rg(dn_in, sn), rg(dm_in, sm)};
    for (const Range &o : outs) {
        for (const Range &i : ins)
            if (overlap(o, i)) return XLSTM_ERR_INVALID_ARG;
        for (const Range &o2 : outs)
            if (&o2 != &o && overlap(o, o2)) return XLSTM_ERR_INVALID_ARG;
    }
    if (desc->chunk != 0 && desc->chunk != 64) return XLSTM_ERR_UNSUPPORTED;
    const size_t need = xlstm_mlstm_bwd_workspace_size(desc);
    if (!workspace || workspace_bytes < need) return XLSTM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return XLSTM_ERR_INVALID_ARG;
    xlstm::BwdArgs a;
    a.B = desc->B; a.H = desc->H; a.T = desc->T; a.dqk = desc->d_qk; a.dv = desc->d_v;
    a.dtype = desc->qkv_dtype; a.scale = desc->qk_scale;
    a.q = q; a.k = k; a.v = v; a.ig = i_pre; a.fg = f_pre; a.C0 = C_in; a.n0 = n_in; a.m0 = m_in;
    a.dh = dh; a.dCT = dC_out; a.dnT = dn_out;
    a.dq = dq; a.dk = dk; a.dv_ = dv; a.di = di_pre; a.df = df_pre; a.dC0 = dC_in; a.dn0 = dn_in; a.dm0 = dm_in;
    a.workspace = workspace;
    if (cudaMemsetAsync(workspace, 0, 16, stream) != cudaSuccess) return XLSTM_ERR_CUDA;
    return xlstm::launch_backward(a, stream) == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}

xlstm_status_t xlstm_mlstm_workspace_status(const void *workspace, int32_t *where,
                                            cudaStream_t stream) {
    if (!workspace) return XLSTM_ERR_INVALID_ARG;
    int32_t blk[4] = {0, 0, 0, 0};
    if (cudaMemcpyAsync(blk, workspace, sizeof(blk), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return XLSTM_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return XLSTM_ERR_CUDA;
    if (where) *where = blk[xlstm::kStatusWhere];
    return static_cast<xlstm_status_t>(blk[xlstm::kStatusCode]);
}

const char *xlstm_status_string(xlstm_status_t s) {
    switch (s) {
        case XLSTM_OK: return "ok";
        case XLSTM_ERR_INVALID_ARG: return "invalid argument";
        case XLSTM_ERR_UNSUPPORTED: return "unsupported configuration";
        case XLSTM_ERR_CUDA: return "CUDA launch error";
        case XLSTM_ERR_TIMEOUT: return "device wait timed out";
        case XLSTM_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

const char *xlstm_mlstm_version(void) { return "xlstm_mlstm_b200 0.1 (sm_100a)"; }

const char *xlstm_mlstm_chunkwise_kernel(const xlstm_mlstm_desc_t *desc) {
    if (!desc || !dims_ok(desc)) return "none";
    if (!chunk_ok(desc)) return "none";
    FwdArgs a = pack(desc, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                     nullptr, nullptr, nullptr, nullptr);
    if (a.T == 0) return "copy";
    return xlstm::chunkwise_tc_supported(a) ? "tcgen05" : "simt";
}

void xlstm_mlstm_test_timeout_next(int32_t enable) { xlstm::set_chunkwise_tc_fault(enable ? 1 : 0); }

}  // extern "C"
