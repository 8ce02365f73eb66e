/*
 * Oracle token-by-expert histogram, prefix scan and permutation.
 *
 * TEST INFRASTRUCTURE (see oracle.h).
 *
 * Batching expert work ("DwarfStar", hysenlabs.com, "Model support and
 * quantisation": Blackwell runs batched expert work on FP4 matrix
 * instructions) needs the (token, slot) pairs grouped by expert. Definition:
 *   slot s = t*k + j (token t's j-th expert idx[s]);
 *   counts[e]   = number of slots routed to e;
 *   offsets     = exclusive prefix sum of counts, offsets[E] = T*k;
 *   perm[row]   = slot, rows of expert e are [offsets[e], offsets[e+1]) in
 *                 ascending slot order (so ascending token order);
 *   inv_perm[s] = the row holding slot s.
 * Returns 0, or -1 if some idx is outside [0, E).
 */
#include <stdlib.h>

#include "oracle.h"

int ora_permute(const int32_t *idx, int T, int k, int E, int32_t *counts, int32_t *offsets,
                int32_t *perm, int32_t *inv_perm) {
    const int64_t S = (int64_t)T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t s = 0; s < S; ++s) {
        if (idx[s] < 0 || idx[s] >= E) return -1;
        counts[idx[s]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (int64_t s = 0; s < S; ++s) {
        const int32_t r = fill[idx[s]]++;
        perm[r] = (int32_t)s;
        inv_perm[s] = r;
    }
    free(fill);
    return 0;
}
