// Sparse map: histogram, exclusive-scan expert offsets and stable slot assignment.
//
// Sources: ScatterMoE guide, "2. Grouped Coordinate Indexing Without Padding" (Histogram(e),
// Offsets(e)); "Add scalable sparse map kernel for large MoE models (128+ experts)", "Pass 1:
// Histogram with Atomics" and "Pass 2: Two Assignment Variants". That page's atomic assignment
// orders slots by atomic arrival and so is not deterministic; its own tests ask for deterministic
// results ("4. Correctness Validation"). Here slots inside an expert follow the flat route index
// (a stable counting sort), which is unique, so the map is bit-exact run to run.
//
// Work split: the route list is cut into units of kUnit consecutive routes, one warp per unit.
//  1. count:  each warp walks its unit 32 routes at a time; __match_any_sync groups the lanes
//             holding the same expert, the group's lowest lane adds the group size to the warp's
//             private shared-memory counter of that expert (no atomics; warp-aggregated). The
//             warp writes its per-expert counts to scratch[unit][e].
//  2. scan:   one block turns scratch into per-(unit, expert) bases: the exclusive prefix over
//             units of each expert plus the expert's offset (the exclusive prefix over experts
//             of the totals), and writes counts and offsets[E+1].
//  3. assign: each warp walks its unit again with its counters preset to the bases; a route's
//             slot is its expert counter plus the number of lower lanes of its match group.
// No kernel waits on another block, so nothing here can spin.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kIters = 16;                // 32-route steps per unit
constexpr int kUnit = 32 * kIters;        // 512 routes per warp
constexpr int kMaxE = 256;

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
map_count_kernel(const int32_t *__restrict__ te, int64_t R, int32_t E, int64_t units,
                 int32_t *__restrict__ unit_counts, unsigned *status) {
    __shared__ int32_t cnt[kWarpsPerBlock][kMaxE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t u = (int64_t)blockIdx.x * kWarpsPerBlock + warp;
    if (u >= units) return;
    for (int e = lane; e < E; e += 32) cnt[warp][e] = 0;
    __syncwarp();
    bool bad = false;
    const int64_t base = u * kUnit;
    int ev[kIters];
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int64_t i = base + it * 32 + lane;
        int e = -1;
        if (i < R) {
            e = __ldg(te + i);
            if (e < 0 || e >= E) {
                bad = true;
                e = -1;
            }
        }
        ev[it] = e;
    }
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int e = ev[it];
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int leader = __ffs(peers) - 1;
        if (e >= 0 && lane == leader) cnt[warp][e] += __popc(peers);
        __syncwarp();
    }
    if (bad) atomicOr(status, kStatusBadExpert);
    for (int e = lane; e < E; e += 32) unit_counts[u * E + e] = cnt[warp][e];
}

// One block of 1024 threads. Thread (g, e): group g of the units, expert e.
__global__ void __launch_bounds__(1024)
map_scan_kernel(int32_t *__restrict__ unit_counts, int64_t units, int32_t E,
                int32_t *__restrict__ counts, int32_t *__restrict__ offsets) {
    __shared__ int32_t part[1024];
    __shared__ int32_t total[kMaxE + 1];
    const int tid = threadIdx.x;
    const int groups = max(1, 1024 / E);
    const int g = tid / E, e = tid % E;
    const bool active = g < groups;
    const int64_t per = (units + groups - 1) / groups;
    const int64_t u0 = active ? ((int64_t)g * per < units ? (int64_t)g * per : units) : 0;
    const int64_t u1 = active ? (u0 + per < units ? u0 + per : units) : 0;
    int32_t sum = 0;
    if (active)
        for (int64_t u = u0; u < u1; ++u) sum += unit_counts[u * E + e];
    part[tid] = sum;
    __syncthreads();
    // exclusive prefix of the groups, per expert; expert totals
    if (tid < E) {
        int32_t run = 0;
        for (int gg = 0; gg < groups; ++gg) {
            const int32_t c = part[gg * E + tid];
            part[gg * E + tid] = run;
            run += c;
        }
        total[tid] = run;
    }
    __syncthreads();
    // exclusive prefix over experts (E <= 256: one thread; negligible next to the loads)
    if (tid == 0) {
        int32_t run = 0;
        for (int ee = 0; ee < E; ++ee) {
            const int32_t c = total[ee];
            counts[ee] = c;
            offsets[ee] = run;
            total[ee] = run;
            run += c;
        }
        offsets[E] = run;
    }
    __syncthreads();
    if (active) {
        int32_t run = total[e] + part[g * E + e];
        for (int64_t u = u0; u < u1; ++u) {
            const int32_t c = unit_counts[u * E + e];
            unit_counts[u * E + e] = run;
            run += c;
        }
    }
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
map_assign_kernel(const int32_t *__restrict__ te, int64_t R, int32_t E, int64_t units,
                  const int32_t *__restrict__ unit_base, int32_t *__restrict__ sparse_rows,
                  int32_t *__restrict__ sorted_rows) {
    __shared__ int32_t cnt[kWarpsPerBlock][kMaxE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t u = (int64_t)blockIdx.x * kWarpsPerBlock + warp;
    if (u >= units) return;
    for (int e = lane; e < E; e += 32) cnt[warp][e] = unit_base[u * E + e];
    __syncwarp();
    const unsigned lower = (1u << lane) - 1u;
    const int64_t base = u * kUnit;
    int ev[kIters];
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int64_t i = base + it * 32 + lane;
        int e = -1;
        if (i < R) {
            e = __ldg(te + i);
            if (e < 0 || e >= E) e = -1;
        }
        ev[it] = e;
    }
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int64_t i = base + it * 32 + lane;
        const int e = ev[it];
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        int32_t slot = -1;
        if (e >= 0) slot = cnt[warp][e] + __popc(peers & lower);
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) cnt[warp][e] += __popc(peers);
        __syncwarp();
        if (i < R) {
            sparse_rows[i] = slot;
            if (slot >= 0) sorted_rows[slot] = (int32_t)i;
        }
    }
}

// The whole map in one block when the routes fit 32 units (R <= 16384): warp w counts unit w
// into cnt[w][e]; the per-expert exclusive prefix over the 32 warps plus the expert offset turns
// cnt into bases; the warps walk their units again and assign stable slots. Same results as the
// three-kernel path, one launch instead of three (the decode and Mixtral-prefill route counts).
constexpr int kSmallUnits = 32;
__global__ void __launch_bounds__(kSmallUnits * 32)
map_small_kernel(const int32_t *__restrict__ te, int64_t R, int32_t E,
                 int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                 int32_t *__restrict__ sparse_rows, int32_t *__restrict__ sorted_rows,
                 unsigned *status) {
    __shared__ int32_t cnt[kSmallUnits][kMaxE];
    __shared__ int32_t eoff[kMaxE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = lane; e < E; e += 32) cnt[warp][e] = 0;
    __syncwarp();
    const int64_t base = (int64_t)warp * kUnit;
    // all of this lane's routes at once: kIters independent loads instead of a dependent chain
    int ev[kIters];
    bool bad = false;
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int64_t i = base + it * 32 + lane;
        int e = -1;
        if (i < R) {
            e = __ldg(te + i);
            if (e < 0 || e >= E) {
                bad = true;
                e = -1;
            }
        }
        ev[it] = e;
    }
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int e = ev[it];
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1) cnt[warp][e] += __popc(peers);
        __syncwarp();
    }
    if (bad) atomicOr(status, kStatusBadExpert);
    __syncthreads();
    // per expert: exclusive prefix over the warps (in place) and the total
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t run = 0;
        for (int w = 0; w < kSmallUnits; ++w) {
            const int32_t c = cnt[w][e];
            cnt[w][e] = run;
            run += c;
        }
        eoff[e] = run;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int32_t run = 0;
        for (int e = 0; e < E; ++e) {
            const int32_t c = eoff[e];
            counts[e] = c;
            offsets[e] = run;
            eoff[e] = run;
            run += c;
        }
        offsets[E] = run;
    }
    __syncthreads();
    for (int e = lane; e < E; e += 32) cnt[warp][e] += eoff[e];
    __syncwarp();
    const unsigned lower = (1u << lane) - 1u;
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int64_t i = base + it * 32 + lane;
        const int e = ev[it];
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        int32_t slot = -1;
        if (e >= 0) slot = cnt[warp][e] + __popc(peers & lower);
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) cnt[warp][e] += __popc(peers);
        __syncwarp();
        if (i < R) {
            sparse_rows[i] = slot;
            if (slot >= 0) sorted_rows[slot] = (int32_t)i;
        }
    }
}

}  // namespace

size_t map_scratch_bytes(int64_t R, int32_t E) {
    const int64_t units = (R + kUnit - 1) / kUnit;
    return (size_t)(units > 0 ? units : 1) * (size_t)E * sizeof(int32_t);
}

int launch_sparse_map(const int32_t *te, int64_t R, int32_t E, int32_t *counts, int32_t *offsets,
                      int32_t *sparse_rows, int32_t *sorted_rows, int32_t *scratch,
                      unsigned *status, cudaStream_t s, int *n_launch) {
    const int64_t units = (R + kUnit - 1) / kUnit;
    const int64_t blocks = (units + kWarpsPerBlock - 1) / kWarpsPerBlock;
    int n = 0;
    if (units <= kSmallUnits) {
        map_small_kernel<<<1, kSmallUnits * 32, 0, s>>>(te, R, E, counts, offsets, sparse_rows,
                                                         sorted_rows, status);
        if (n_launch) *n_launch += 1;
        return 0;
    }
    if (blocks > 0) {
        map_count_kernel<<<(unsigned)blocks, kWarpsPerBlock * 32, 0, s>>>(te, R, E, units,
                                                                          scratch, status);
        ++n;
    }
    map_scan_kernel<<<1, 1024, 0, s>>>(scratch, units, E, counts, offsets);
    ++n;
    if (blocks > 0) {
        map_assign_kernel<<<(unsigned)blocks, kWarpsPerBlock * 32, 0, s>>>(
            te, R, E, units, scratch, sparse_rows, sorted_rows);
        ++n;
    }
    if (n_launch) *n_launch += n;
    return 0;
}

}  // namespace moe
