// Grid schedule of the router (k_route): how query blocks group into runs
// (one CTA each) and how the runs map to CTA indices.  Pure index arithmetic,
// shared by the kernel and its launcher; plain C++ as well as CUDA, so the
// CPU tests compile it too.
#pragma once

#ifdef __CUDACC__
#define HGA_HD __host__ __device__ __forceinline__
#else
#define HGA_HD inline
#endif

namespace hga {

// Run length for the grid: CTAs = ceil(NB / n) runs x Hkv x B.  When the
// grid fits in one wave of resident CTAs, take the n that minimises the
// query blocks of the busiest SM (its CTA count times n), ties to the longer
// run (fewer reads of the chunk table); otherwise the longest run.  Every
// block's routing is computed the same way whatever run it falls in, so n
// changes the schedule, never a result.
inline int pick_run(int NB, int units, int nmax, int sms, int per_sm) {
    const long long slots = (long long)sms * per_sm;
    int best = nmax;
    long long best_cost = -1;
    for (int n = nmax; n >= 1; --n) {
        const long long ctas = (long long)((NB + n - 1) / n) * units;
        if (ctas > slots) break;                      // shorter runs only add CTAs
        const long long cost = (long long)n * ((ctas + sms - 1) / sms);
        if (best_cost < 0 || cost < best_cost) {
            best = n;
            best_cost = cost;
        }
    }
    return best;
}

// Run and (KV head, sequence) unit of the CTA at linear index lin, for R
// runs per unit and U units.  Chunk-scoring work grows with the run index
// (a later run has more middle chunks), and CTAs start about in linear order,
// two to an SM.  So the lightest run is paired with the heaviest, the next
// lightest with the next heaviest, and so on; the two members of pair i sit
// at linear indices i and i + N/2, and which of them takes the heavy run
// alternates with i, so that CTAs adjacent in linear order and CTAs N/2
// apart both hold complementary work.  With N odd the median CTA comes last.
HGA_HD void pair_slot(int lin, int R, int U, int *run, int *unit) {
    const int N = R * U, P = N / 2;
    int j;                                     // position in run-major order
    if (lin >= 2 * P) {
        j = P;
    } else {
        const int i = lin < P ? lin : lin - P;
        const bool heavy = ((i & 1) == 0) == (lin < P);
        j = heavy ? N - 1 - i : i;
    }
    *run = j / U;
    *unit = j % U;
}

}  // namespace hga
