// sz_internal.h -- launcher interface between the C ABI layer and the kernels.
// Host arrays are read during the call only (copied into kernel parameters).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "splitzip.h"

namespace sz {

struct PlanArgs {
    int dtype, T, num_sms;
    const void *const *in;
    const uint64_t *n;
    uint32_t *ctl, *hist, *ticket;
    uint8_t *plans;
    const sz_paged_t *paged;  // T input page descriptors, or null (contiguous inputs)
};

struct EncodeArgs {
    int dtype, T, num_sms;
    const uint8_t *plans;
    const void *const *in;
    const uint64_t *n;
    void *const *out;
    const size_t *cap;
    uint32_t *ctl;
    unsigned long long *status;
    unsigned long long *group;
    unsigned long long *totals;  // may be null
    int reuse;                   // codebook reuse: plans give codebooks only
    const sz_paged_t *paged;     // T input page descriptors, or null (contiguous inputs)
};

struct DecodeArgs {
    int dtype, T, num_sms;
    const void *const *comp;
    const size_t *comp_bytes;
    void *const *out;
    const uint64_t *n;
    uint32_t *ctl;
    const sz_paged_t *paged;  // T output page descriptors, or null (contiguous outputs)
};

// Host checks of an encode call (contiguous or paged inputs; the pools of
// paged ones in d_in) against the workspace at d_ws: SZ_OK, or the status the
// call returns without enqueuing anything.
sz_status check_encode_args(sz_dtype dtype, int T, const sz_plan_t *d_plans, const void *const *d_in,
                            const uint64_t *n, void *const *d_out, const size_t *out_cap, const uint64_t *d_totals,
                            const void *d_ws, size_t ws_bytes);

// Kernel page reference of descriptor d (or a contiguous tensor when d is null).
PageRef page_ref(const sz_paged_t *d);

sz_status launch_plan(const PlanArgs &a, cudaStream_t stream);
sz_status launch_encode(const EncodeArgs &a, cudaStream_t stream);
sz_status launch_decode(const DecodeArgs &a, cudaStream_t stream);

}  // namespace sz
