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
    // LMOE_OPT_Z_RECHECK_DELTA: margin of z's exact re-rounding, zcheck_delta * (1 + 0.4 |z|);
    // >= 4x the largest fp32 error of z measured at Ultra width with fc1 in chunks of 4 k-blocks
    // (1.16e-6 + 0.45e-6 |z| over 524288 elements; the smallest ratio seen is 4.5)
    float zcheck_delta = 6e-6f;
    // LMOE_OPT_ACT_RECHECK_TAU: relu2 activations with h above this are re-rounded exactly when
    // within the accumulation-error margin act_c0 + act_c1 h of a bf16 midpoint. The margin is the
    // largest fp32 error measured at K = 8192 in TMEM chunks of 8 k-blocks; the shared up GEMM
    // (K = H = 8192) runs in chunks of 4 (measured on fc1, the same x and K: 1.16e-6 + 0.45e-6 h,
    // so the margin is 1.4-2x), the expert up GEMM (K = L = 2048) has a quarter of the chunks
    float act_tau = 2.0f;
    float act_c0 = (float)lmoe::kActC0, act_c1 = (float)lmoe::kActC1;
    unsigned spin_limit = 1u << 24;
    int num_sms = 148;
    int launches = 0;                  // kernels launched by the last call
    int last_cuda_error = 0;           // cudaError_t of the last runtime call that failed (0: none yet)
    void* const* prof_events = nullptr;  // latentmoe_set_profile_events
    int prof_n = 0;
    // second stream of a forward: the routing tail runs on it next to the exact re-roundings,
    // forked from and joined back into the caller's stream by the two events
    cudaStream_t aux = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
};
