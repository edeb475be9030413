// mlstm_api.cu -- the C ABI of libmlstm: argument checks, workspace layout, dispatch.
//
// Every entry point checks its arguments on the host before it enqueues
// anything, returns a status code and never throws.  Kernels are enqueued on
// the caller's stream; nothing here synchronizes except mlstm_fwd_status.
#include "mlstm.h"
#include "mlstm_internal.h"
#include "tc_fwd.h"

#include <stdint.h>

using namespace mlstm;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool dims_ok_fwd(int DHQK, int DHV)
{
    return DHQK >= 8 && DHQK <= 512 && DHQK % 8 == 0 && DHV >= 8 && DHV <= 512 && DHV % 8 == 0;
}

bool chunk_ok(int chunk) { return chunk == 16 || chunk == 32 || chunk == 64 || chunk == 128; }

// Lays out the workspace (base may be NULL to size it).  Returns the bytes used.
size_t plan_workspace(char *base, int BH, int S, int DHQK, int DHV, int chunk, bool bf16, FwdWorkspace *w)
{
    FwdWorkspace tmp;
    if (!w) w = &tmp;
    const int NC = (S + chunk - 1) / chunk;
    w->NC = NC;
    size_t off = 0;
    auto take = [&](size_t bytes) -> char * {
        char *p = base ? base + off : nullptr;
        off = align_up(off + bytes, 256);
        return p;
    };
    w->status = reinterpret_cast<uint32_t *>(take(sizeof(uint32_t)));
    w->A = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * S));
    w->M = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * S));
    w->G = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * NC));
    w->Bc = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * NC));
    w->MC = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * (NC + 1)));
    w->tc = tc_path_supported(bf16, DHQK, DHV, chunk) && S > 0;
    w->CS = w->NS = w->GP = w->SGb = w->DC = w->DN = nullptr;
    w->CS16 = nullptr;
    w->NSEG = 0;
    w->R = 0;
    if (w->tc) {
        const int nseg = tc_num_segments(BH, DHV, NC);
        w->R = (NC + nseg - 1) / nseg;
        w->NSEG = (NC + w->R - 1) / w->R;
        w->GP = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * NC));
        w->SGb = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * w->NSEG * 2));
        w->DC = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * w->NSEG * DHQK * DHV));
        w->DN = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * w->NSEG * DHQK));
    } else {
        w->CS = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * NC * DHQK * DHV));
        w->NS = reinterpret_cast<float *>(take(sizeof(float) * (size_t)BH * NC * DHQK));
    }
    return off;
}

mlstm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA; }

// Lays out the backward pass's workspace (base may be NULL to size it).  Returns the bytes used.
size_t plan_bwd_workspace(char *base, int BH, int S, int DHQK, int DHV, int chunk, bool tc, BwdWorkspace *w)
{
    BwdWorkspace tmp;
    if (!w) w = &tmp;
    const int NC = (S + chunk - 1) / chunk;
    const int NTK = (DHQK + 31) / 32;
    w->NC = NC;
    size_t off = 0;
    auto take = [&](size_t bytes) -> char * {
        char *p = base ? base + off : nullptr;
        off = align_up(off + bytes, 256);
        return p;
    };
    const size_t f = sizeof(float);
    w->status = reinterpret_cast<uint32_t *>(take(sizeof(uint32_t)));
    w->A = reinterpret_cast<float *>(take(f * BH * S));
    w->M = reinterpret_cast<float *>(take(f * BH * S));
    w->G = reinterpret_cast<float *>(take(f * BH * NC));
    w->Bc = reinterpret_cast<float *>(take(f * BH * NC));
    w->MC = reinterpret_cast<float *>(take(f * BH * (NC + 1)));
    // (the tensor-core path keeps the chunk-start states only as their bf16 parts, below)
    w->CS = tc ? nullptr : reinterpret_cast<float *>(take(f * BH * NC * DHQK * DHV));
    w->NS = reinterpret_cast<float *>(take(f * BH * NC * DHQK));
    w->GS = tc ? nullptr : reinterpret_cast<float *>(take(f * BH * NC * DHQK * DHV));
    w->GN = reinterpret_cast<float *>(take(f * BH * NC * DHQK));
    // (the tensor-core path keeps g, dS and A only as bf16 parts or copies, below)
    w->Gt = tc ? nullptr : reinterpret_cast<float *>(take(f * BH * S * DHV));
    w->DD = reinterpret_cast<float *>(take(f * BH * S));
    w->P2 = tc ? nullptr : reinterpret_cast<float *>(take(f * BH * NC * chunk * chunk));
    w->AI = tc ? nullptr : reinterpret_cast<float *>(take(f * BH * NC * chunk * chunk));
    w->QD = reinterpret_cast<float *>(take(f * BH * S * NTK));
    w->KD = reinterpret_cast<float *>(take(f * BH * S * NTK));
    w->KI = reinterpret_cast<float *>(take(f * BH * S * NTK));
    w->RECT = reinterpret_cast<float *>(take(f * BH * S));
    w->NEP = tc ? 4 * (DHQK / 128) * (DHV / 64) : 1;
    w->EP = reinterpret_cast<float *>(take(f * BH * NC * w->NEP));
    w->DEN = reinterpret_cast<float *>(take(f * BH * S));
    w->NRM = reinterpret_cast<float *>(take(f * BH * S));
    w->DOTP = reinterpret_cast<float *>(take(f * BH * S * ((DHV + 63) / 64)));
    w->tc = tc;
    w->CS16 = w->GS16 = w->Gt16 = w->P216 = w->AI16 = w->SG16 = w->WK16 = nullptr;
    if (tc) {
        const size_t h = sizeof(__nv_bfloat16);
        w->CS16 = reinterpret_cast<__nv_bfloat16 *>(take(2 * h * BH * NC * DHQK * DHV));   // two parts
        w->GS16 = reinterpret_cast<__nv_bfloat16 *>(take(h * BH * NC * DHQK * DHV));
        w->Gt16 = reinterpret_cast<__nv_bfloat16 *>(take(2 * h * BH * S * DHV));             // two parts
        w->P216 = reinterpret_cast<__nv_bfloat16 *>(take(h * BH * NC * chunk * chunk));
        w->AI16 = reinterpret_cast<__nv_bfloat16 *>(take(2 * h * BH * NC * chunk * chunk));   // two parts
        w->SG16 = reinterpret_cast<__nv_bfloat16 *>(take(2 * h * BH * S * DHV));             // two parts
        w->WK16 = reinterpret_cast<__nv_bfloat16 *>(take(2 * h * BH * S * DHQK));            // two parts
    }
    return off;
}

}  // namespace

extern "C" const char *mlstm_status_string(mlstm_status s)
{
    switch (s) {
    case MLSTM_OK: return "ok";
    case MLSTM_ERR_INVALID_ARG: return "invalid argument (NULL pointer, negative size or misaligned pointer)";
    case MLSTM_ERR_UNSUPPORTED: return "unsupported shape, chunk or dtype";
    case MLSTM_ERR_WORKSPACE: return "workspace missing or too small";
    case MLSTM_ERR_CUDA: return "CUDA launch or runtime error";
    case MLSTM_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    }
    return "unknown status";
}

extern "C" size_t mlstm_fwd_workspace_size(int B, int NH, int S, int DHQK, int DHV, int chunk, mlstm_dtype dt)
{
    if (B < 0 || NH < 0 || S < 0 || (dt != MLSTM_F32 && dt != MLSTM_BF16)) return 0;
    if (!dims_ok_fwd(DHQK, DHV) || !chunk_ok(chunk)) return 0;
    // the limits mlstm_fwd applies: larger shapes are unsupported (and B * NH would overflow)
    if ((long long)B * NH > (1LL << 30) || (long long)S * DHV > (1LL << 40)) return 0;
    return plan_workspace(nullptr, B * NH, S, DHQK, DHV, chunk, dt == MLSTM_BF16, nullptr);
}

extern "C" int mlstm_fwd_kernel_launches(int B, int NH, int S, int DHQK, int DHV, int chunk, mlstm_dtype dt)
{
    if (mlstm_fwd_workspace_size(B, NH, S, DHQK, DHV, chunk, dt) == 0) return 0;
    if (B == 0 || NH == 0 || S == 0) return 0;
    // gate preprocessing (1 or 2) + (segment sums, segment scan, walk) or (carry walk, outputs)
    const int NC = (S + chunk - 1) / chunk;
    return gate_prep_launches(S, NC) + (tc_path_supported(dt == MLSTM_BF16, DHQK, DHV, chunk) ? 3 : 2);
}

extern "C" int mlstm_fwd_tensor_path(int DHQK, int DHV, int chunk, mlstm_dtype dt)
{
    if (dt != MLSTM_F32 && dt != MLSTM_BF16) return -1;
    if (!dims_ok_fwd(DHQK, DHV) || !chunk_ok(chunk)) return -1;
    return tc_path_supported(dt == MLSTM_BF16, DHQK, DHV, chunk) ? 1 : 0;
}

extern "C" int mlstm_fwd_paired_walk(int DHQK, int DHV, int chunk, mlstm_dtype dt)
{
    if (mlstm_fwd_tensor_path(DHQK, DHV, chunk, dt) != 1) return -1;
    return tcfwd::walk_pair_supported(DHQK, DHV, chunk) ? 1 : 0;
}

extern "C" int mlstm_fwd_segments(int B, int NH, int S, int DHQK, int DHV, int chunk, mlstm_dtype dt)
{
    if (B < 0 || NH < 0 || S < 0 || mlstm_fwd_tensor_path(DHQK, DHV, chunk, dt) != 1) return 0;
    if ((long long)B * NH > (1LL << 30) || B * NH == 0 || S == 0) return 0;
    FwdWorkspace w;
    plan_workspace(nullptr, B * NH, S, DHQK, DHV, chunk, true, &w);
    return w.NSEG;
}

namespace {

mlstm_status fwd_impl(const void *q, const void *k, const void *v, const float *igate, const float *fgate,
                      const void *ogate, mlstm_dtype dt, int B, int NH, int S, int DHQK, int DHV, int chunk,
                      const float *C0, const float *n0, const float *m0,
                      void *h_out, float *C_final, float *n_final, float *m_final, void *workspace,
                      size_t workspace_bytes, void *stream, void *const *events, bool outputs = true)
{
    if (B < 0 || NH < 0 || S < 0) return MLSTM_ERR_INVALID_ARG;
    if (dt != MLSTM_F32 && dt != MLSTM_BF16) return MLSTM_ERR_UNSUPPORTED;
    if (!dims_ok_fwd(DHQK, DHV) || !chunk_ok(chunk)) return MLSTM_ERR_UNSUPPORTED;
    if ((long long)B * NH > (1LL << 30) || (long long)S * DHV > (1LL << 40)) return MLSTM_ERR_UNSUPPORTED;
    const int BH = B * NH;
    const bool has_tokens = BH > 0 && S > 0;
    if (has_tokens && outputs) {
        if (!q || !k || !v || !igate || !fgate || !h_out) return MLSTM_ERR_INVALID_ARG;
        const void *ptrs[] = {q, k, v, igate, fgate, h_out};
        for (const void *p : ptrs)
            if (!aligned16(p)) return MLSTM_ERR_INVALID_ARG;
        if (ogate && !aligned16(ogate)) return MLSTM_ERR_INVALID_ARG;
    }
    if (has_tokens && !outputs) {   // the final state only: q, ogate and h are not used
        if (!k || !v || !igate || !fgate) return MLSTM_ERR_INVALID_ARG;
        const void *ptrs[] = {k, v, igate, fgate};
        for (const void *p : ptrs)
            if (!aligned16(p)) return MLSTM_ERR_INVALID_ARG;
    }
    if ((C_final && !aligned16(C_final)) || (n_final && !aligned16(n_final)) || (m_final && !aligned16(m_final)))
        return MLSTM_ERR_INVALID_ARG;
    const bool has_state = C0 || n0 || m0;
    if (has_state && BH > 0) {   // the initial state comes whole or not at all
        if (!C0 || !n0 || !m0) return MLSTM_ERR_INVALID_ARG;
        if (!aligned16(C0) || !aligned16(n0) || !aligned16(m0)) return MLSTM_ERR_INVALID_ARG;
    }
    const bool bf16 = dt == MLSTM_BF16;
    const size_t need = plan_workspace(nullptr, BH, S, DHQK, DHV, chunk, bf16, nullptr);
    if (!workspace || workspace_bytes < need) return MLSTM_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLSTM_ERR_INVALID_ARG;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    FwdWorkspace w;
    plan_workspace(static_cast<char *>(workspace), BH, S, DHQK, DHV, chunk, bf16, &w);
    cudaError_t e = cudaSuccess;
    if (BH == 0 || S == 0) {   // no kernel runs: reset the status word here (else the first gate kernel does)
        e = cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st);
        if (e != cudaSuccess) return MLSTM_ERR_CUDA;
    }
    if (BH == 0) return MLSTM_OK;
    if (S == 0) {   // no tokens: the final state is the initial one (zero state by default)
        const size_t bC = sizeof(float) * (size_t)BH * DHQK * DHV, bn = sizeof(float) * (size_t)BH * DHQK,
                     bm = sizeof(float) * (size_t)BH;
        if (has_state) {
            if (C_final && C_final != C0) e = cudaMemcpyAsync(C_final, C0, bC, cudaMemcpyDeviceToDevice, st);
            if (e == cudaSuccess && n_final && n_final != n0)
                e = cudaMemcpyAsync(n_final, n0, bn, cudaMemcpyDeviceToDevice, st);
            if (e == cudaSuccess && m_final && m_final != m0)
                e = cudaMemcpyAsync(m_final, m0, bm, cudaMemcpyDeviceToDevice, st);
        } else {
            if (C_final) e = cudaMemsetAsync(C_final, 0, bC, st);
            if (e == cudaSuccess && n_final) e = cudaMemsetAsync(n_final, 0, bn, st);
            if (e == cudaSuccess && m_final) e = cudaMemsetAsync(m_final, 0, bm, st);
        }
        return cuda_status(e);
    }

    PhaseMark mark;
    mark.events = events;
    mark.stream = st;
    if (mark(0) != cudaSuccess) return MLSTM_ERR_CUDA;
    GatePrepArgs gp{igate, fgate, BH, S, chunk, w.NC, w.A, w.M, w.G, w.Bc, w.MC, w.R, w.NSEG, w.GP, w.SGb, m0, w.status,
                    st};
    e = launch_gate_prep(gp);
    if (e != cudaSuccess) return MLSTM_ERR_CUDA;
    if (mark(1) != cudaSuccess) return MLSTM_ERR_CUDA;
    FwdArgs fa{q, k, v, ogate, igate, fgate, h_out, C_final, n_final, m_final, C0, n0, BH, S, DHQK, DHV, chunk,
               dt == MLSTM_BF16, st, outputs};
    e = w.tc ? launch_fwd_tc(fa, w, mark) : launch_fwd_simt(fa, w, mark);
    if (e != cudaSuccess) return MLSTM_ERR_CUDA;
    return cuda_status(mark(MLSTM_FWD_PHASES));
}

}  // namespace

extern "C" {

mlstm_status mlstm_fwd(const void *q, const void *k, const void *v, const float *igate, const float *fgate,
                       const void *ogate, mlstm_dtype dt, int B, int NH, int S, int DHQK, int DHV, int chunk,
                       void *h_out, float *C_final, float *n_final, float *m_final, void *workspace,
                       size_t workspace_bytes, void *stream)
{
    return fwd_impl(q, k, v, igate, fgate, ogate, dt, B, NH, S, DHQK, DHV, chunk, nullptr, nullptr, nullptr, h_out,
                    C_final, n_final, m_final, workspace, workspace_bytes, stream, nullptr);
}

mlstm_status mlstm_fwd_final_state(const void *k, const void *v, const float *igate, const float *fgate,
                                   mlstm_dtype dt, int B, int NH, int S, int DHQK, int DHV, int chunk,
                                   float *C_final, float *n_final, float *m_final, void *workspace,
                                   size_t workspace_bytes, void *stream)
{
    return fwd_impl(nullptr, k, v, igate, fgate, nullptr, dt, B, NH, S, DHQK, DHV, chunk, nullptr, nullptr, nullptr,
                    nullptr, C_final, n_final, m_final, workspace, workspace_bytes, stream, nullptr, false);
}

mlstm_status mlstm_fwd_state(const void *q, const void *k, const void *v, const float *igate, const float *fgate,
                             const void *ogate, mlstm_dtype dt, int B, int NH, int S, int DHQK, int DHV, int chunk,
                             const float *C0, const float *n0, const float *m0, void *h_out, float *C_final,
                             float *n_final, float *m_final, void *workspace, size_t workspace_bytes, void *stream)
{
    return fwd_impl(q, k, v, igate, fgate, ogate, dt, B, NH, S, DHQK, DHV, chunk, C0, n0, m0, h_out, C_final,
                    n_final, m_final, workspace, workspace_bytes, stream, nullptr);
}

mlstm_status mlstm_fwd_profiled(const void *q, const void *k, const void *v, const float *igate,
                                const float *fgate, const void *ogate, mlstm_dtype dt, int B, int NH, int S,
                                int DHQK, int DHV, int chunk, void *h_out, float *C_final, float *n_final,
                                float *m_final, void *workspace, size_t workspace_bytes, void *stream,
                                void *const *events)
{
    if (!events) return MLSTM_ERR_INVALID_ARG;     // entries may be NULL: those boundaries are not recorded
    return fwd_impl(q, k, v, igate, fgate, ogate, dt, B, NH, S, DHQK, DHV, chunk, nullptr, nullptr, nullptr, h_out,
                    C_final, n_final, m_final, workspace, workspace_bytes, stream, events);
}

mlstm_status mlstm_fwd_status(const void *workspace, void *stream)
{
    if (!workspace) return MLSTM_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return MLSTM_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return MLSTM_ERR_CUDA;
    return word == 0 ? MLSTM_OK : MLSTM_ERR_TIMEOUT;
}

mlstm_status mlstm_step(float *C, float *n, float *m, const void *q, const void *k, const void *v,
                        const float *igate, const float *fgate, const void *ogate, mlstm_dtype dt, int B, int NH,
                        int DHQK, int DHV, void *h_out, void *stream)
{
    if (B < 0 || NH < 0) return MLSTM_ERR_INVALID_ARG;
    if (dt != MLSTM_F32 && dt != MLSTM_BF16) return MLSTM_ERR_UNSUPPORTED;
    if (DHQK < 8 || DHQK > 512 || DHQK % 8 || DHV < 4 || DHV > 1024 || DHV % 4) return MLSTM_ERR_UNSUPPORTED;
    if ((long long)B * NH > (1LL << 30)) return MLSTM_ERR_UNSUPPORTED;
    const int BH = B * NH;
    if (BH == 0) return MLSTM_OK;
    if (!C || !n || !m || !q || !k || !v || !igate || !fgate || !h_out) return MLSTM_ERR_INVALID_ARG;
    const void *ptrs[] = {C, n, m, q, k, v, igate, fgate, h_out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return MLSTM_ERR_INVALID_ARG;
    if (ogate && !aligned16(ogate)) return MLSTM_ERR_INVALID_ARG;
    StepArgs a{C, n, m, q, k, v, ogate, igate, fgate, h_out, BH, DHQK, DHV, dt == MLSTM_BF16,
               reinterpret_cast<cudaStream_t>(stream)};
    return cuda_status(launch_step(a));
}

}  // extern "C"

extern "C" size_t mlstm_bwd_workspace_size(int B, int NH, int S, int DHQK, int DHV, int chunk, mlstm_dtype dt)
{
    if (B < 0 || NH < 0 || S < 0 || (dt != MLSTM_F32 && dt != MLSTM_BF16)) return 0;
    if (!dims_ok_fwd(DHQK, DHV) || !chunk_ok(chunk)) return 0;
    if ((long long)B * NH > (1LL << 30) || (long long)S * DHV > (1LL << 40)) return 0;
    return plan_bwd_workspace(nullptr, B * NH, S, DHQK, DHV, chunk, bwd_tc_path(dt == MLSTM_BF16, B * NH, S, DHQK, DHV, chunk),
                              nullptr);
}

extern "C" int mlstm_bwd_tensor_path(int DHQK, int DHV, int chunk, mlstm_dtype dt)
{
    if ((dt != MLSTM_F32 && dt != MLSTM_BF16) || !dims_ok_fwd(DHQK, DHV) || !chunk_ok(chunk)) return -1;
    return bwd_tc_path(dt == MLSTM_BF16, 1, chunk, DHQK, DHV, chunk) ? 1 : 0;
}

extern "C" mlstm_status mlstm_bwd(const void *q, const void *k, const void *v, const float *igate, const float *fgate,
                                  const void *ogate, const void *dh, mlstm_dtype dt, int B, int NH, int S, int DHQK,
                                  int DHV, int chunk, void *dq, void *dk, void *dv, float *digate, float *dfgate,
                                  void *dogate, void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 0 || NH < 0 || S < 0) return MLSTM_ERR_INVALID_ARG;
    if (dt != MLSTM_F32 && dt != MLSTM_BF16) return MLSTM_ERR_UNSUPPORTED;
    if (!dims_ok_fwd(DHQK, DHV) || !chunk_ok(chunk)) return MLSTM_ERR_UNSUPPORTED;
    if ((long long)B * NH > (1LL << 30) || (long long)S * DHV > (1LL << 40)) return MLSTM_ERR_UNSUPPORTED;
    const int BH = B * NH;
    if (BH == 0 || S == 0) return MLSTM_OK;   // no tokens: every gradient is empty
    const void *ins[] = {q, k, v, igate, fgate, dh, dq, dk, dv, digate, dfgate};
    for (const void *p : ins)
        if (!p || !aligned16(p)) return MLSTM_ERR_INVALID_ARG;
    if (ogate && (!dogate || !aligned16(ogate) || !aligned16(dogate))) return MLSTM_ERR_INVALID_ARG;
    const bool bf16 = dt == MLSTM_BF16;
    const bool tc = bwd_tc_path(bf16, BH, S, DHQK, DHV, chunk);
    const size_t need = plan_bwd_workspace(nullptr, BH, S, DHQK, DHV, chunk, tc, nullptr);
    if (!workspace || workspace_bytes < need) return MLSTM_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLSTM_ERR_INVALID_ARG;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    BwdWorkspace w;
    plan_bwd_workspace(static_cast<char *>(workspace), BH, S, DHQK, DHV, chunk, tc, &w);
    // gate preprocessing and the chunk-start states of the forward pass (its fp32 carry)
    GatePrepArgs gp{igate, fgate, BH, S, chunk, w.NC, w.A, w.M, w.G, w.Bc, w.MC, 0, 0, nullptr, nullptr, nullptr,
                    w.status, st};
    if (launch_gate_prep(gp) != cudaSuccess) return MLSTM_ERR_CUDA;
    FwdWorkspace fw{};
    fw.status = w.status;
    fw.NC = w.NC;
    fw.A = w.A; fw.M = w.M; fw.G = w.G; fw.Bc = w.Bc; fw.MC = w.MC;
    fw.CS = w.CS; fw.NS = w.NS; fw.CS16 = w.CS16;
    fw.tc = false;
    FwdArgs fa{q, k, v, nullptr, igate, fgate, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, BH, S, DHQK, DHV,
               chunk, bf16, st, false};
    // (on the tensor-core path the backward's own carry walk computes the chunk-start states)
    if (!w.tc && launch_fwd_simt(fa, fw, PhaseMark{}) != cudaSuccess) return MLSTM_ERR_CUDA;
    BwdArgs ba{q, k, v, ogate, dh, igate, fgate, dq, dk, dv, dogate, digate, dfgate, BH, S, DHQK, DHV, chunk, bf16,
               st};
    return cuda_status(launch_bwd(ba, w));
}
