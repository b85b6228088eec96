// kernels.h -- internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace hgrn2 {

struct SimtFwdArgs {
    const void *q, *lf, *x;
    const float *h0;
    void *o;
    float *hT;
    int B, T, H, dk, dv, C;
};

struct SimtBwdArgs {
    const void *q, *lf, *x, *dO;
    const float *h0, *dhT;
    void *dq, *dlf, *dx;
    float *dh0;
    float *rs;   // [B*H*dk] workspace: rowsum(dhT * hT)
    int B, T, H, dk, dv, C;
};

size_t simt_fwd_smem(int C, int dk, int dv);
size_t simt_bwd_dq_smem(int C, int dk, int dv);
size_t simt_bwd_rev_smem(int C, int dk, int dv);
cudaError_t launch_simt_fwd(const SimtFwdArgs &a, bool bf16, cudaStream_t st);
cudaError_t launch_simt_bwd(const SimtBwdArgs &a, bool bf16, cudaStream_t st);

cudaError_t launch_step(const void *q, const void *lf, const void *x, float *S, void *o, int B, int H,
                        int dk, int dv, bool bf16, cudaStream_t st);

}  // namespace hgrn2
