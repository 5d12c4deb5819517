// Definition of the opaque coli_moe handle (internal).
#pragma once

#include <cuda.h>

#include "coli_internal.cuh"

struct coli_moe {
    int device;
    int H, I, E, k, n_shared;
    int prefill_min;             // 0: grouped GEMM unless the fused decode kernel takes the call
    int per_row;                 // one scale per row (COLI_GROUP_PER_ROW) instead of gs64
    int num_sms;
    coli::DevExpert* d_experts;  // device table, E + n_shared entries
    CUtensorMap* d_wmaps;        // packed-code tensor maps, 3 per expert (tensor-core path)
    CUtensorMap* d_bmaps;        // 128-byte-wide swizzled code maps, 3 per expert (small batches)
    CUtensorMap* d_dmaps;        // swizzled 3-D code maps, 3 per expert (fused decode path)
};
