// qmv_inst_umma.cu -- tensor-memory (tcgen05) affine qmv kernels: bits x the
// accumulator read width MLD (the power of two >= M), bf16 x.
#include "qmv_launch.cuh"
#include "qmv_umma.cuh"

namespace qmv {

namespace {

template <int B, int MLD>
cudaError_t launch_umma_t(const Params& p, const UmmaParams& u, const Launch& L) {
    static std::atomic<unsigned> configured{0};
    auto kern = qmv_umma_kernel<B, MLD>;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned bit = 1u << (dev & 31);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = L.grid;
    cfg.blockDim = L.block;
    cfg.dynamicSmemBytes = L.smem;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)u.S;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
    if (L.pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, p, u);
}

template <int B, int MLD>
cudaError_t clusters_t(const UmmaParams& u, size_t smem, int* out) {
    auto kern = qmv_umma_kernel<B, MLD>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)u.S, 1, 1);
    cfg.blockDim = dim3(320, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)u.S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaOccupancyMaxActiveClusters(out, kern, &cfg);
}

template <int B>
cudaError_t dispatch_mld(int mld, const Params& p, const UmmaParams& u, const Launch& L) {
    switch (mld) {
        case 1: return launch_umma_t<B, 1>(p, u, L);
        case 2: return launch_umma_t<B, 2>(p, u, L);
        case 4: return launch_umma_t<B, 4>(p, u, L);
        case 8: return launch_umma_t<B, 8>(p, u, L);
        case 16: return launch_umma_t<B, 16>(p, u, L);
        case 32: return launch_umma_t<B, 32>(p, u, L);
        case 64: return launch_umma_t<B, 64>(p, u, L);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_umma_affine(int bits, int mld, const Params& p, const UmmaParams& u, const Launch& L) {
    switch (bits) {
        case 2: return dispatch_mld<2>(mld, p, u, L);
        case 3: return dispatch_mld<3>(mld, p, u, L);
        case 4: return dispatch_mld<4>(mld, p, u, L);
        case 5: return dispatch_mld<5>(mld, p, u, L);
        case 6: return dispatch_mld<6>(mld, p, u, L);
        case 8: return dispatch_mld<8>(mld, p, u, L);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t umma_max_clusters(int bits, const UmmaParams& u, size_t smem, int* out) {
    // the occupancy of one instantiation stands for all (same block, smem)
    switch (bits) {
        case 2: return clusters_t<2, 1>(u, smem, out);
        case 3: return clusters_t<3, 1>(u, smem, out);
        case 4: return clusters_t<4, 1>(u, smem, out);
        case 5: return clusters_t<5, 1>(u, smem, out);
        case 6: return clusters_t<6, 1>(u, smem, out);
        case 8: return clusters_t<8, 1>(u, smem, out);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qmv
