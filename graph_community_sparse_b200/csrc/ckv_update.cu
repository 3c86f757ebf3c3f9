// Local community update for a newly generated token, sm_100a: the
// stand-alone kernel (ckv_assign_update, ckv_append_assign).  The update of
// one graph unit, and where it comes from in the pages, is in ckv_assign.cuh;
// the attention's merge kernel runs the same code when the step is fused.
#include <math.h>

#include "ckv_assign.cuh"

namespace ckv {

// One block per graph unit, one warp per candidate (see assign_unit).
template <typename T, int D>
__global__ void __launch_bounds__(CKV_NEIGHBOURS * 32) assign_kernel(AssignParams p) {
    __shared__ int s_nbr[CKV_NEIGHBOURS];
    __shared__ __align__(16) AssignScratch<D> s_scratch;
    pdl_wait();  // everything this kernel reads may come from the kernel before it
    const int u = blockIdx.x;
    if (threadIdx.x < CKV_NEIGHBOURS) s_nbr[threadIdx.x] = p.nbr8[(size_t)u * CKV_NEIGHBOURS + threadIdx.x];
    __syncthreads();
    assign_unit<T, D, CKV_NEIGHBOURS, true>(p, u, s_nbr, threadIdx.x, s_scratch, [] { __syncthreads(); });
}

cudaError_t launch_assign_update(const CacheView& c, const GraphView& g, int pos, const void* k_new,
                                 const void* v_new, const int32_t* nbr8, int32_t* assigned, cudaStream_t st) {
    const AssignParams p = make_assign_params(c, g, pos, k_new, v_new, nbr8, assigned);
    if (p.U <= 0) return cudaSuccess;
    const dim3 grid(p.U), block(CKV_NEIGHBOURS * 32);
    if (c.dtype == CKV_DTYPE_BF16) {
        if (c.d == 128) return launch_pdl(KK_UPDATE, assign_kernel<__nv_bfloat16, 128>, grid, block, 0, st, p);
        return launch_pdl(KK_UPDATE, assign_kernel<__nv_bfloat16, 64>, grid, block, 0, st, p);
    }
    if (c.d == 128) return launch_pdl(KK_UPDATE, assign_kernel<float, 128>, grid, block, 0, st, p);
    return launch_pdl(KK_UPDATE, assign_kernel<float, 64>, grid, block, 0, st, p);
}

}  // namespace ckv
