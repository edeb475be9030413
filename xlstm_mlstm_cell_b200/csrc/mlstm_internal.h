// mlstm_internal.h -- launch descriptors shared by the host side of libmlstm.
#pragma once

#include <cuda_bf16.h>
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
    int R, NSEG;             // segments of R chunks (tensor-core path; NSEG = 0 otherwise)
    float *GP, *SGb;         // [BH][NC] in-segment prefix of chunk decays, [BH][NSEG][2] segment maps
    const float *m0;         // [BH] initial stabilizer, NULL = 0
    uint32_t *status;        // bounded-wait status word, reset to 0 by the first gate kernel
    cudaStream_t stream;
};

struct FwdArgs {
    const void *q, *k, *v, *ogate;
    const float *igate, *fgate;
    void *h;
    float *C_final, *n_final, *m_final;
    const float *C0, *n0;    // initial state [BH][DHQK][DHV], [BH][DHQK]; NULL = zero
    int BH, S, DHQK, DHV, chunk;
    bool bf16;
    cudaStream_t stream;
    bool outputs;            // false: the final state only (no output stage; q, ogate, h unused)
};

// Device workspace of one mlstm_fwd call, carved from the caller's buffer.
struct FwdWorkspace {
    uint32_t *status;      // bounded-wait status word (0 = fine)
    int NC;                // chunks
    float *A, *M;          // [BH][S] chunk-local cumulative log decay and prefix maximum of i~ - a
    float *G, *Bc;         // [BH][NC] chunk log decay, chunk max-plus offset
    float *MC;             // [BH][NC+1] stabilizer at chunk starts (last = final m)
    float *CS, *NS;        // SIMT path: state at every chunk start
    __nv_bfloat16 *CS16;   // optional bf16 parts of CS [BH][NC][2][DHQK][DHV] (the backward), else NULL
    // tensor-core path
    bool tc;               // the tensor-core path is used
    int NSEG, R;           // segments per head and chunks per segment
    float *GP;             // [BH][NC] sum of the decays of the earlier chunks of the same segment
    float *SGb;            // [BH][NSEG][2] segment max-plus map (total log decay G, offset b)
    float *DC;             // [BH][NSEG][DHQK/4][DHV][4] segment contributions, then segment start states
    float *DN;             // [BH][NSEG][DHQK] same for the normalizer
};

struct BwdArgs {
    const void *q, *k, *v, *ogate, *dh;
    const float *igate, *fgate;
    void *dq, *dk, *dv, *dogate;
    float *digate, *dfgate;
    int BH, S, DHQK, DHV, chunk;
    bool bf16;
    cudaStream_t stream;
};

// Device workspace of one mlstm_bwd call.
struct BwdWorkspace {
    uint32_t *status;
    int NC;
    float *A, *M, *G, *Bc, *MC;   // gate preprocessing, as for the forward pass
    float *CS, *NS;               // forward chunk-start states [BH][NC][DHQK][DHV], [BH][NC][DHQK]
    float *GS, *GN;               // state gradients per chunk, same layouts
    float *Gt;                    // [BH][S][DHV] gradient of the read-out numerator
    float *DD;                    // [BH][S] gradient of the denominator
    float *P2, *AI;               // [BH][NC][chunk][chunk] score gradients and scores
    // [BH][S][ceil(DHQK / 32)] partial q . dq^inter, k . dk and k . dk^inter (^inter: the term of the
    // tokens of other chunks, through the chunk's state or state gradient)
    float *QD, *KD, *KI;
    float *RECT;                  // [BH][S] sum of dA_ts A_ts over the pairs s < j <= t of j's chunk
    float *EP;                    // [BH][NC][NEP] partial sums of E_c, the pairs that skip chunk c
    int NEP;                      // 1 on the CUDA-core path, 4 (DHQK / 128) (DHV / 64) on the tensor-core path
    float *DEN, *NRM;             // [BH][S] read-out denominator and its floored magnitude
    float *DOTP;                  // [BH][S][ceil(DHV / 64)] partial row sums of g . hh
    // the tensor-core path (bf16 inputs, bwd_tc_path; there CS, GS, Gt, P2 and AI are NULL): the
    // chunk-end state gradients and dS as bf16 (layouts of GS, P2), the chunk-start states, the
    // scores ([BH][NC][2][...]) and g ([BH][2][S][DHV]) as two bf16 parts each (value and rounding
    // residue); NULL on the CUDA-core path
    bool tc;
    __nv_bfloat16 *CS16, *GS16, *Gt16, *P216, *AI16;
    __nv_bfloat16 *SG16;          // sc_t g_t as two bf16 parts [BH][2][S][DHV]
    __nv_bfloat16 *WK16;          // w_s k_s as two bf16 parts [BH][2][S][DHQK] (the carry walk)
};

// Records the caller's phase events (mlstm_fwd_profiled); a no-op without events.
struct PhaseMark {
    void *const *events = nullptr;
    cudaStream_t stream = nullptr;
    cudaError_t operator()(int phase) const
    {
        return events && events[phase] ? cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[phase]), stream)
                                       : cudaSuccess;
    }
};

cudaError_t launch_step(const StepArgs &a);
cudaError_t launch_gate_prep(const GatePrepArgs &a);
int gate_prep_launches(int S, int NC);   // kernels launch_gate_prep launches for S tokens, NC chunks per head
cudaError_t launch_fwd_simt(const FwdArgs &a, const FwdWorkspace &w, const PhaseMark &mark);
size_t simt_state_bytes(int BH, int NC, int DHQK, int DHV);
bool tc_path_supported(bool bf16, int DHQK, int DHV, int chunk);
int tc_num_segments(int BH, int DHV, int NC);
cudaError_t launch_fwd_tc(const FwdArgs &a, const FwdWorkspace &w, const PhaseMark &mark);
cudaError_t launch_bwd(const BwdArgs &a, const BwdWorkspace &w);
// The backward's dq, dk and dv products run on the tensor cores for these arguments.
bool bwd_tc_path(bool bf16, int BH, int S, int DHQK, int DHV, int chunk);

}  // namespace mlstm
