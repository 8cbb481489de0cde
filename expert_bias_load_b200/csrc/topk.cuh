// topk.cuh -- per-thread running Top-K over one token's experts.
//
// Order: larger key first; on equal keys the lower expert index first
// ("SMEBU Load Balancing", eq. (17) selects Top-K of s + b; the pages leave
// ties open and this library breaks them toward the lower index).  Experts are
// pushed in increasing index order, so a strict comparison keeps an earlier
// (lower-index) expert ahead of a later one with an equal key.
#pragma once

#include <cmath>
#include <cstdint>

namespace ebl {

template <int K>
struct RowTopK {
    float key[K];
    float score[K];
    int idx[K];

    __device__ __forceinline__ void init() {
#pragma unroll
        for (int k = 0; k < K; ++k) {
            key[k] = -INFINITY;
            score[k] = 0.0f;
            idx[k] = 0x7fffffff;
        }
    }

    // Offer expert `i` (i larger than every index offered before).
    __device__ __forceinline__ void push(float kv, float s, int i) {
        if (kv > key[K - 1]) {
            key[K - 1] = kv;
            score[K - 1] = s;
            idx[K - 1] = i;
#pragma unroll
            for (int p = K - 1; p > 0; --p) {
                const bool up = key[p] > key[p - 1];
                const float tk = key[p], ts = score[p];
                const int ti = idx[p];
                key[p] = up ? key[p - 1] : tk;
                score[p] = up ? score[p - 1] : ts;
                idx[p] = up ? idx[p - 1] : ti;
                key[p - 1] = up ? tk : key[p - 1];
                score[p - 1] = up ? ts : score[p - 1];
                idx[p - 1] = up ? ti : idx[p - 1];
            }
        }
    }
};

}  // namespace ebl
