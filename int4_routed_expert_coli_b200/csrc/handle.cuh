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
    CUtensorMap* d_bmaps;        // small-batch maps, 6 per expert: codes (128-byte swizzled
                                 // boxes) and scales (8 x 128 boxes; zero where not used)
    CUtensorMap* d_dmaps;        // swizzled 3-D code maps, 3 per expert (fused decode path)
};
