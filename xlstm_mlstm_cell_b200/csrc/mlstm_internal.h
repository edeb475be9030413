// mlstm_internal.h -- launch descriptors shared by the host side of libmlstm.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mlstm {

struct StepArgs {
    float *C, *n, *m;
    const void *q, *k, *v, *ogate;
    const float *igate, *fgate;
    void *h;
    int BH, DHQK, DHV;
    bool bf16;
    cudaStream_t stream;
};

struct GatePrepArgs {
    const float *igate, *fgate;
    int BH, S, L, NC;
    float *A, *M, *G, *Bc, *MC;
    cudaStream_t stream;
};

struct FwdArgs {
    const void *q, *k, *v, *ogate;
    const float *igate, *fgate;
    void *h;
    float *C_final, *n_final, *m_final;
    int BH, S, DHQK, DHV, chunk;
    bool bf16;
    cudaStream_t stream;
};

// Device workspace of one mlstm_fwd call, carved from the caller's buffer.
struct FwdWorkspace {
    uint32_t *status;      // bounded-wait status word (0 = fine)
    int NC;                // chunks
    float *A, *M;          // [BH][S] chunk-local cumulative log decay, per-token stabilizer
    float *G, *Bc;         // [BH][NC] chunk log decay, chunk max-plus offset
    float *MC;             // [BH][NC+1] stabilizer at chunk starts (last = final m)
    float *CS, *NS;        // SIMT path: state at every chunk start
    // tensor-core path
    int NSEG, R;           // segments and chunks per segment
    float *SA, *SG, *SB;   // [BH][NSEG] segment log decay, max-plus offset (tensor-core path)
    float *SM;             // [BH][NSEG+1] stabilizer at segment starts
    float *DC;             // [BH][NSEG][DHQK][DHV] segment contributions (fp32)
    float *DN;             // [BH][NSEG][DHQK]
    float *SC;             // [BH][NSEG][DHQK][DHV] state at segment starts (fp32)
    float *SN;             // [BH][NSEG][DHQK]
};

// Records the caller's phase events (mlstm_fwd_profiled); a no-op without events.
struct PhaseMark {
    void *const *events = nullptr;
    cudaStream_t stream = nullptr;
    cudaError_t operator()(int phase) const
    {
        return events ? cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[phase]), stream) : cudaSuccess;
    }
};

cudaError_t launch_step(const StepArgs &a);
cudaError_t launch_gate_prep(const GatePrepArgs &a);
cudaError_t launch_fwd_simt(const FwdArgs &a, const FwdWorkspace &w, const PhaseMark &mark);
size_t simt_state_bytes(int BH, int NC, int DHQK, int DHV);

}  // namespace mlstm
