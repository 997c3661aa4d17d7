// qmv_inst_tcg.cuh -- launch table of the per-group tensor-core ring kernels
// for one x dtype (included by qmv_inst_tcg_{bf16,f16}.cu only).
#pragma once

#include "qmv_launch.cuh"
#include "qmv_tcg.cuh"

namespace qmv {

template <class T, int G, int NT>
static cudaError_t launch_tcg_t(const Params& p, const Launch& L) {
    static std::atomic<unsigned> cfg{0};
    return launch_kernel(qmv_tcg_kernel<T, G, NT>, cfg, L, p);
}

template <class T, int G>
static cudaError_t launch_tcg_n(int nt, const Params& p, const Launch& L) {
    switch (nt) {
        case 1: return launch_tcg_t<T, G, 1>(p, L);
        case 2: return launch_tcg_t<T, G, 2>(p, L);
        case 4: return launch_tcg_t<T, G, 4>(p, L);
        default: return cudaErrorInvalidValue;
    }
}

template <class T>
static cudaError_t launch_tcg_g(int G, int nt, const Params& p, const Launch& L) {
    switch (G) {
        case 32: return launch_tcg_n<T, 32>(nt, p, L);
        case 64: return launch_tcg_n<T, 64>(nt, p, L);
        case 128: return launch_tcg_n<T, 128>(nt, p, L);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qmv
