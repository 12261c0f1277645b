// handle.h -- host-side state of a LatentMoE layer handle.
#pragma once
#include "lmoe_internal.h"

struct lmoe_handle {
    lmoe_config cfg;
    lmoe_weights w;
    int* herr = nullptr;       // pinned, device-mapped error word (host view)
    int* derr = nullptr;       // same word, device view
    int gemm_path = 0;         // lmoe_option LMOE_OPT_GEMM_PATH
    int fp64_all = 0;          // LMOE_OPT_ROUTER_FP64_ALL
    float flag_delta = 2e-5f;  // LMOE_OPT_FLAG_DELTA (10x the largest fp32 score error seen at Ultra width, x2)
    float zcheck_delta = 5e-6f;  // LMOE_OPT_Z_RECHECK_DELTA (mean |fp32 - exact| of z: ~3e-7)
    unsigned spin_limit = 1u << 24;
    int num_sms = 148;
    int launches = 0;                  // kernels launched by the last call
    int last_cuda_error = 0;           // cudaError_t of the last runtime call that failed (0: none yet)
    void* const* prof_events = nullptr;  // latentmoe_set_profile_events
    int prof_n = 0;
};
