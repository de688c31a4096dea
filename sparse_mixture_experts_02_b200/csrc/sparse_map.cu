// Sparse map: histogram, exclusive-scan expert offsets and stable slot assignment.
//
// Sources: ScatterMoE guide, "2. Grouped Coordinate Indexing Without Padding" (Histogram(e),
// Offsets(e)); "Add scalable sparse map kernel for large MoE models (128+ experts)", "Pass 1:
// Histogram with Atomics" and "Pass 2: Two Assignment Variants". That page's atomic assignment
// orders slots by atomic arrival and so is not deterministic; its own tests ask for deterministic
// results ("4. Correctness Validation"). Here slots inside an expert follow the flat route index
// (a stable counting sort), which is unique, so the map is bit-exact run to run.
//
// Work split: the route list is cut into units of consecutive routes, one warp per unit, eight
// units per block. A unit is 512 routes (16 steps of 32) when that still gives at least one block
// per SM; below that (the 10^4-10^5 routes of a forward) it shrinks to 256, 128, 64 or 32 routes
// so that the grid keeps about one to two blocks per SM instead of leaving most SMs idle.
//  1. count:  each warp counts its unit into its own shared-memory counters (shared atomics);
//             the block sums its warps and writes its per-expert counts to scratch,
//             expert-major: bcount[e][block].
//  2. scan:   one block per expert turns its row of block counts into exclusive bases (prefix
//             over the blocks) and writes the expert's total.
//  3. assign: each block forms the expert offsets (exclusive prefix of the totals), recounts its
//             routes and gives each its stable slot, in one of two forms chosen by the table size
//             per route: with at most 8 experts per route a lane owns (E <= 8 IT), each lane
//             owns consecutive routes and keeps a byte counter per expert in shared memory
//             (map_assign_lane_kernel); with more, each lane takes one route per 32-route step
//             and finds its same-expert neighbours with ballots (map_assign_warp_kernel). Paired
//             at 2^24-2^26 routes, the lane form took 0.76-0.80 of the warp form's time at 8 and
//             64 experts, 0.95 at 128 and 1.14-1.17 at 256; at the 2^15-2^17 routes of a forward
//             (1 or 2 routes a lane) 1.11-1.13 at 128 and 256 experts.
// Every kernel is grid-parallel and no block waits on another, so nothing here can spin; the
// scratch is E x (blocks + 1) words, one eighth of a per-warp layout.
#include "moe_internal.cuh"

#include <algorithm>
#include <mutex>

namespace moe {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kIters = 16;                // 32-route steps per unit
constexpr int kUnit = 32 * kIters;        // 512 routes per warp
constexpr int kMaxE = 256;
constexpr int kScanThreads = 1024;
constexpr int kScanPer = 8;               // rows of 32 block counts a warp (rows scan)
constexpr int64_t kScanRowsFrom = 2048;   // block counts above which that scan is used

// Lanes of the warp holding the same value as this lane, v < 2^nbits: the intersection over the
// value's bits of the lanes that agree with it on that bit.
__device__ __forceinline__ unsigned same_value_lanes(unsigned v, int nbits) {
    unsigned m = 0xffffffffu;
    for (int bit = 0; bit < nbits; ++bit) {
        const unsigned b = (v >> bit) & 1u;
        const unsigned ones = __ballot_sync(0xffffffffu, b);
        m &= b ? ones : ~ones;
    }
    return m;
}

// Bits that hold expert ids 0..E (E itself stands for "no expert").
__device__ __forceinline__ int id_bits(int32_t E) { return 32 - __clz(E); }

// Loads the IT x 32 routes of a warp's unit (-1 past R or for an id outside [0, E)).
template <int IT>
__device__ __forceinline__ bool load_unit(const int32_t *__restrict__ te, int64_t R, int32_t E,
                                          int64_t base, int lane, int (&ev)[IT]) {
    bool bad = false;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
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
    return bad;
}

// Adds the unit's routes to the warp's per-expert counters. Counting needs no order, so plain
// shared-memory atomics do it (measured 1.3-1.5x faster than warp-aggregating with ballots).
template <int IT>
__device__ __forceinline__ void count_unit(const int (&ev)[IT], int32_t *cnt) {
#pragma unroll
    for (int it = 0; it < IT; ++it)
        if (ev[it] >= 0) atomicAdd(&cnt[ev[it]], 1);
    __syncwarp();
}

template <int IT>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
map_count_kernel(const int32_t *__restrict__ te, int64_t R, int32_t E, int64_t nblk,
                 int32_t *__restrict__ bcount, unsigned *status) {
    constexpr int UNIT = 32 * IT, BLOCK_ROUTES = UNIT * kWarpsPerBlock;
    __shared__ int32_t cnt[kWarpsPerBlock][kMaxE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.x;
    for (int e = lane; e < E; e += 32) cnt[warp][e] = 0;
    __syncwarp();
    int ev[IT];
    const bool bad = load_unit<IT>(te, R, E, b * BLOCK_ROUTES + (int64_t)warp * UNIT, lane, ev);
    count_unit<IT>(ev, cnt[warp]);
    if (bad) atomicOr(status, kStatusBadExpert);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t sum = 0;
#pragma unroll
        for (int w = 0; w < kWarpsPerBlock; ++w) sum += cnt[w][e];
        bcount[(int64_t)e * nblk + b] = sum;
    }
}

// Exclusive prefix of v over the block's NT threads (blockDim.x == NT); *total gets the block's
// sum. `wsum` holds NT / 32 words of shared memory.
template <int NT>
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t *wsum, int32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t inc = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, inc, d);
        if (lane >= d) inc += t;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int32_t w = lane < NT / 32 ? wsum[lane] : 0;
        int32_t winc = w;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, winc, d);
            if (lane >= d) winc += t;
        }
        if (lane < NT / 32) wsum[lane] = winc - w;  // exclusive over warps
        if (lane == 31) *total = winc;
    }
    __syncthreads();
    const int32_t ex = wsum[warp] + inc - v;
    __syncthreads();  // wsum is reused by the next call
    return ex;
}

// One block per expert: its row of block counts becomes exclusive bases; totals[e] = the sum.
// One entry per thread and pass: the form for up to kScanRowsFrom block counts, where one or two
// passes of three barriers are all the latency there is (map_scan_rows_kernel below took 2-4 us
// longer at the 128-192 blocks of a 128- or 64-expert forward).
__global__ void __launch_bounds__(kScanThreads)
map_scan_kernel(int32_t *__restrict__ bcount, int64_t nblk, int32_t *__restrict__ totals) {
    __shared__ int32_t wsum[kScanThreads / 32];
    __shared__ int32_t chunk_total;
    int32_t *row = bcount + (int64_t)blockIdx.x * nblk;
    int32_t carry = 0;
    for (int64_t c = 0; c < nblk; c += kScanThreads) {
        const int64_t j = c + threadIdx.x;
        const int32_t v = j < nblk ? row[j] : 0;
        const int32_t ex = block_exclusive_scan<kScanThreads>(v, wsum, &chunk_total);
        if (j < nblk) row[j] = carry + ex;
        carry += chunk_total;
        __syncthreads();
    }
    if (threadIdx.x == 0) totals[blockIdx.x] = carry;
}

// The scan for more than kScanRowsFrom block counts. A pass covers kScanThreads x kScanPer
// entries: warp w takes kScanPer consecutive rows of 32 entries, loads them coalesced (one entry a
// lane per row), scans each row with shuffles and carries the row totals along; one block-wide
// scan of the warp totals then offsets the warps, and the stores are coalesced the same way. 32
// registers keep two blocks on an SM (256 experts in one wave); the 16384 blocks of 2^26 routes
// take two passes, where a scan of one entry per thread ran 16 passes of three barriers (19 us at
// eight experts).
__global__ void __launch_bounds__(kScanThreads, 2)
map_scan_rows_kernel(int32_t *__restrict__ bcount, int64_t nblk, int32_t *__restrict__ totals) {
    __shared__ int32_t wsum[kScanThreads / 32];
    __shared__ int32_t chunk_total;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t *row = bcount + (int64_t)blockIdx.x * nblk;
    int32_t carry = 0;
    for (int64_t c = 0; c < nblk; c += (int64_t)kScanThreads * kScanPer) {
        const int64_t j0 = c + (int64_t)warp * 32 * kScanPer + lane;
        int32_t v[kScanPer];
#pragma unroll
        for (int q = 0; q < kScanPer; ++q) v[q] = j0 + 32 * q < nblk ? row[j0 + 32 * q] : 0;
        // exclusive prefix of the warp's 32 x kScanPer entries, in registers
        int32_t wrun = 0;
#pragma unroll
        for (int q = 0; q < kScanPer; ++q) {
            int32_t inc = v[q];
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int32_t t = __shfl_up_sync(0xffffffffu, inc, d);
                if (lane >= d) inc += t;
            }
            v[q] = wrun + inc - v[q];
            wrun += __shfl_sync(0xffffffffu, inc, 31);
        }
        // the warps' totals: one value per warp into the block scan (lane 0 carries it)
        const int32_t wex =
            block_exclusive_scan<kScanThreads>(lane == 0 ? wrun : 0, wsum, &chunk_total);
        const int32_t off = carry + __shfl_sync(0xffffffffu, wex, 0);
#pragma unroll
        for (int q = 0; q < kScanPer; ++q)
            if (j0 + 32 * q < nblk) row[j0 + 32 * q] = off + v[q];
        carry += chunk_total;
        __syncthreads();  // chunk_total is rewritten by the next pass
    }
    if (threadIdx.x == 0) totals[blockIdx.x] = carry;
}

// Assign, one route per lane: each warp walks its unit 32 routes at a time; a route's slot is its
// expert counter plus the number of lower lanes holding the same expert, found with one ballot per
// bit of the id (a warp multisplit: the lanes that agree on every bit; measured faster than
// __match_any_sync at 64 and 256 experts), and the lowest of those lanes advances the counter.
// Its cost grows with log2(E) per route, where map_assign_lane_kernel's grows with E per warp: it
// serves the many-expert shapes (E > 8 routes per lane). All of a block's global loads (the
// expert totals, its block bases, the warps' routes) are issued before any of them is used: with
// few blocks per SM, three dependent load phases left the kernel waiting on memory latency (ncu:
// long-scoreboard stalls first, 24% warps active).
template <int IT>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 4)
map_assign_warp_kernel(const int32_t *__restrict__ te, int64_t R, int32_t E, int64_t nblk,
                  const int32_t *__restrict__ bbase, const int32_t *__restrict__ totals,
                  int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                  int32_t *__restrict__ sparse_rows, int32_t *__restrict__ sorted_rows,
                  unsigned *status) {
    constexpr int NT = kWarpsPerBlock * 32;
    constexpr int UNIT = 32 * IT, BLOCK_ROUTES = UNIT * kWarpsPerBlock;
    static_assert(NT == kMaxE, "one thread per expert");
    __shared__ int32_t cnt[kWarpsPerBlock][kMaxE];
    __shared__ int32_t wsum[NT / 32];
    __shared__ int32_t total, btotal;
    __shared__ int32_t s_first[kMaxE], s_pre[kMaxE];  // per expert: first slot, staging offset
    __shared__ int32_t stage_r[BLOCK_ROUTES];          // routes, grouped by expert
    __shared__ uint8_t stage_e[BLOCK_ROUTES];          // their experts
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e_t = threadIdx.x;  // this thread's expert in the per-expert steps
    const int64_t b = blockIdx.x;
    const int32_t tot_e = e_t < E ? __ldg(totals + e_t) : 0;
    const int32_t bb_e = e_t < E ? __ldg(bbase + (int64_t)e_t * nblk + b) : 0;
    int ev[IT];
    const int64_t base = b * BLOCK_ROUTES + (int64_t)warp * UNIT;
    load_unit<IT>(te, R, E, base, lane, ev);
    // expert offsets: exclusive prefix of the totals
    const int32_t eoff_e = block_exclusive_scan<NT>(tot_e, wsum, &total);
    if (b == 0) {
        if (e_t < E) {
            counts[e_t] = tot_e;
            offsets[e_t] = eoff_e;
        }
        if (threadIdx.x == 0) offsets[E] = total;
    }
    // recount this block's units per warp
    for (int e = lane; e < E; e += 32) cnt[warp][e] = 0;
    __syncwarp();
    count_unit<IT>(ev, cnt[warp]);
    __syncthreads();
    // per expert: expert offset + block base, then exclusive prefix over the block's warps
    int32_t bcount_e = 0;
    if (e_t < E) {
        int32_t run = eoff_e + bb_e;
#pragma unroll
        for (int w = 0; w < kWarpsPerBlock; ++w) {
            const int32_t c = cnt[w][e_t];
            cnt[w][e_t] = run;
            run += c;
        }
        bcount_e = run - (eoff_e + bb_e);
    }
    // the block's slots of expert e are the contiguous range [first, first + bcount_e). With more
    // than 16 experts a warp's 32 routes spread over many experts and a direct sorted_rows store
    // is one scattered word per route: the routes are then staged in shared memory, expert after
    // expert, and written out contiguously below (measured 22% faster at 2^26 routes and 64 or
    // 256 experts, 10% slower at 8, where a warp's stores already form runs of about four).
    const bool staged = E > 16;
    const int32_t pre_e = block_exclusive_scan<NT>(bcount_e, wsum, &btotal);
    if (e_t < E) {
        s_first[e_t] = eoff_e + bb_e;
        s_pre[e_t] = pre_e;
    }
    __syncthreads();
    // stable slots
    const unsigned lower = (1u << lane) - 1u;
    const int nbits = id_bits(E);
    int32_t *wc = cnt[warp];
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int64_t i = base + it * 32 + lane;
        const int e = ev[it];
        const unsigned peers = same_value_lanes(e >= 0 ? (unsigned)e : (unsigned)E, nbits);
        int32_t slot = -1;
        if (e >= 0) slot = wc[e] + __popc(peers & lower);
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) wc[e] += __popc(peers);
        __syncwarp();
        if (i < R) {
            sparse_rows[i] = slot;
            if (slot >= 0) {
                if (staged) {
                    const int32_t local = s_pre[e] + (slot - s_first[e]);
                    if (dev::debug_in_range(local, BLOCK_ROUTES, status)) {
                        stage_r[local] = (int32_t)i;
                        stage_e[local] = (uint8_t)e;
                    }
                } else if (dev::debug_in_range(slot, R, status)) {
                    sorted_rows[slot] = (int32_t)i;
                }
            }
        }
    }
    if (!staged) return;  // uniform over the block
    __syncthreads();
    // sorted_rows: consecutive threads write consecutive slots of one expert's range
    for (int j = threadIdx.x; j < btotal; j += NT) {
        const int e = stage_e[j];
        const int64_t slot = (int64_t)s_first[e] + (j - s_pre[e]);
        if (dev::debug_in_range(slot, R, status)) sorted_rows[slot] = stage_r[j];
    }
}

// Shared memory of map_assign_lane_kernel, sized by E (W = kWarpsPerBlock, B = block routes):
//   tab   [W][E][32] u8   per warp and expert, one byte per lane: the lane's routes of that
//                         expert, then their exclusive prefix inside the lane's half-warp
//   stage [B]        u32  the block's routes grouped by expert, in slot order: the route's offset
//                         in the block (bits 0-15) and its expert (bits 16-23)
//   base  [W][2][E]  u16  staging position of the first route of the expert in the warp's lower
//                         or upper half-warp (before that: the warp's and the lower half's counts)
//   delta [E]        i32  slot minus staging position, per expert
template <int IT>
struct AssignSmem {
    static constexpr int B = kWarpsPerBlock * 32 * IT;
    static constexpr size_t W = kWarpsPerBlock;
    __host__ __device__ static size_t stage(int E) { return W * E * 32; }
    __host__ __device__ static size_t base(int E) { return stage(E) + (size_t)B * 4; }
    __host__ __device__ static size_t delta(int E) { return base(E) + W * 2 * E * 2; }
    __host__ __device__ static size_t bytes(int E) { return delta(E) + (size_t)E * 4; }
};

// Stable slots of the block's routes. Each lane owns IT consecutive routes of its warp's unit, so
// the order of routes is (warp, lane, position in the lane), and a route's place among the
// block's routes of its expert is the sum of
//   - the expert's routes in the lower warps and, for lanes 16-31, in lanes 0-15 (base),
//   - its routes in the lower lanes of the same half-warp (the byte-packed prefix of tab),
//   - the lane's earlier routes of the expert (the count the lane had when it reached the route).
// Counting is a plain read-increment-write of the lane's own byte (no atomics, no ballots); the
// prefix over 16 lanes adds four counts per 32-bit word with one multiply (the bytes stay below
// 256: at most 15 x 16 routes before the last lane of a half). The block's routes are staged in
// shared memory expert after expert and written to sorted_rows in contiguous runs. All of a
// block's global loads are issued before any of them is used. Under ncu at 2^24 routes and eight
// experts the shared-memory pipe is the busiest unit: 87% with two staging stores and four shared
// loads per route in the slot step, 75% with the one packed store and three loads here.
template <int IT>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 2)
map_assign_lane_kernel(const int32_t *__restrict__ te, int64_t R, int32_t E, int64_t nblk,
                       const int32_t *__restrict__ bbase, const int32_t *__restrict__ totals,
                       int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                       int32_t *__restrict__ sparse_rows, int32_t *__restrict__ sorted_rows,
                       unsigned *status) {
    constexpr int NT = kWarpsPerBlock * 32;
    constexpr int UNIT = 32 * IT;
    using L = AssignSmem<IT>;
    constexpr int BLOCK_ROUTES = L::B;
    static_assert(NT == kMaxE, "one thread per expert");
    static_assert(IT <= 16, "a half-warp prefix of byte counts stays below 256");
    static_assert(BLOCK_ROUTES <= 65536, "a route's offset in the block fits 16 bits");
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t *tab = smem;
    uint32_t *stage = reinterpret_cast<uint32_t *>(smem + L::stage(E));
    uint16_t *base = reinterpret_cast<uint16_t *>(smem + L::base(E));
    int32_t *delta = reinterpret_cast<int32_t *>(smem + L::delta(E));
    __shared__ int32_t wsum[NT / 32];
    __shared__ int32_t total, btotal;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e_t = threadIdx.x;  // this thread's expert in the per-expert steps
    const int64_t b = blockIdx.x;
    const int64_t first = b * BLOCK_ROUTES;
    const int32_t tot_e = e_t < E ? __ldg(totals + e_t) : 0;
    const int32_t bb_e = e_t < E ? __ldg(bbase + (int64_t)e_t * nblk + b) : 0;
    // this lane's IT consecutive routes (-1 past R or for an id outside [0, E))
    const int off0 = warp * UNIT + lane * IT;  // offset of the lane's first route in the block
    const int64_t i0 = first + off0;
    const bool full = i0 + IT <= R;
    const bool vec = IT % 4 == 0 && full && (reinterpret_cast<uintptr_t>(te) & 15) == 0;
    int v[IT];
    if (vec) {
#pragma unroll
        for (int q = 0; q < IT / 4; ++q) {
            const int4 t = __ldg(reinterpret_cast<const int4 *>(te + i0) + q);
            v[4 * q] = t.x;
            v[4 * q + 1] = t.y;
            v[4 * q + 2] = t.z;
            v[4 * q + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < IT; ++j) v[j] = i0 + j < R ? __ldg(te + i0 + j) : -1;
    }
#pragma unroll
    for (int j = 0; j < IT; ++j)
        if (v[j] < 0 || v[j] >= E) v[j] = -1;  // the count kernel has flagged it
    // clear the count table
    {
        uint4 *t4 = reinterpret_cast<uint4 *>(tab);
        const int n4 = kWarpsPerBlock * E * 2;
        for (int q = threadIdx.x; q < n4; q += NT) t4[q] = make_uint4(0u, 0u, 0u, 0u);
    }
    // expert offsets: exclusive prefix of the totals (its barriers also order the clearing)
    const int32_t eoff_e = block_exclusive_scan<NT>(tot_e, wsum, &total);
    if (b == 0) {
        if (e_t < E) {
            counts[e_t] = tot_e;
            offsets[e_t] = eoff_e;
        }
        if (threadIdx.x == 0) offsets[E] = total;
    }
    // 1. count: the lane's own byte per expert; the count before a route is its rank in the lane
    uint8_t *tw = tab + (size_t)warp * E * 32 + lane;
#pragma unroll
    for (int j = 0; j < IT; ++j) {
        if (v[j] >= 0) {
            uint8_t *c = tw + v[j] * 32;
            const int r = *c;
            *c = (uint8_t)(r + 1);
            v[j] |= r << 16;
        }
    }
    __syncthreads();
    // 2. per (warp, expert) row: exclusive prefix over each half-warp's 16 lanes, in place; the
    //    lower half's count and the warp's count go to base[w][1][e] and base[w][0][e]
    for (int row = threadIdx.x; row < kWarpsPerBlock * E; row += NT) {
        uint4 *rp = reinterpret_cast<uint4 *>(tab + (size_t)row * 32);
        uint4 h[2] = {rp[0], rp[1]};
        uint32_t half_total[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t carry = 0;
            uint32_t *wd = reinterpret_cast<uint32_t *>(&h[hh]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t x = wd[q];
                wd[q] = x * 0x01010100u + carry * 0x01010101u;  // byte k: carry + bytes 0..k-1
                carry += (x * 0x01010101u) >> 24;               // + the word's four counts
            }
            half_total[hh] = carry;
        }
        rp[0] = h[0];
        rp[1] = h[1];
        const int w = row / E, e = row - w * E;
        base[(w * 2 + 1) * E + e] = (uint16_t)half_total[0];
        base[(w * 2) * E + e] = (uint16_t)(half_total[0] + half_total[1]);
    }
    __syncthreads();
    // 3. per expert: block count, prefix over the warps, staging offset and slot delta
    int32_t bcount_e = 0;
    if (e_t < E) {
#pragma unroll
        for (int w = 0; w < kWarpsPerBlock; ++w) {
            const int32_t c = base[(w * 2) * E + e_t];
            base[(w * 2) * E + e_t] = (uint16_t)bcount_e;
            bcount_e += c;
        }
    }
    const int32_t pre_e = block_exclusive_scan<NT>(bcount_e, wsum, &btotal);
    if (e_t < E) {
#pragma unroll
        for (int w = 0; w < kWarpsPerBlock; ++w) {
            const int32_t lo = base[(w * 2) * E + e_t] + pre_e;
            base[(w * 2) * E + e_t] = (uint16_t)lo;
            base[(w * 2 + 1) * E + e_t] = (uint16_t)(lo + base[(w * 2 + 1) * E + e_t]);
        }
        delta[e_t] = eoff_e + bb_e - pre_e;
    }
    __syncthreads();
    // 4. slots: stage each route at its place in the block's expert-grouped order
    const uint8_t *tcol = tab + (size_t)warp * E * 32 + lane;
    const uint16_t *bw = base + (warp * 2 + (lane >= 16 ? 1 : 0)) * E;
#pragma unroll
    for (int j = 0; j < IT; ++j) {
        int32_t slot = -1;
        if (v[j] >= 0) {
            const int e = v[j] & 0xffff;
            const int32_t pos = (int32_t)bw[e] + (int32_t)tcol[e * 32] + (v[j] >> 16);
            slot = pos + delta[e];
            if (dev::debug_in_range(pos, BLOCK_ROUTES, status))
                stage[pos] = (uint32_t)(off0 + j) | ((uint32_t)e << 16);
        }
        v[j] = slot;
    }
    if (vec && (reinterpret_cast<uintptr_t>(sparse_rows) & 15) == 0) {
#pragma unroll
        for (int q = 0; q < IT / 4; ++q)
            reinterpret_cast<int4 *>(sparse_rows + i0)[q] =
                make_int4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < IT; ++j)
            if (i0 + j < R) sparse_rows[i0 + j] = v[j];
    }
    __syncthreads();
    // 5. sorted_rows: consecutive threads write consecutive slots of one expert's run
    for (int j = threadIdx.x; j < btotal; j += NT) {
        const uint32_t st = stage[j];
        const int64_t slot = (int64_t)j + delta[st >> 16];
        if (dev::debug_in_range(slot, R, status))
            sorted_rows[slot] = (int32_t)(first + (st & 0xffffu));
    }
}

// The whole map in one block when the routes fit 32 units of 512 (R <= 16384). The block has
// just as many warps as the routes need: w = ceil(R / (32 IT)) <= 32 warps of IT steps of 32
// routes, IT the smallest power of two that keeps w <= 32 (a decode batch of 256 routes runs 8
// warps of one step; 32 warps of 16 steps ran every step of every warp, with barriers and
// __match_any_sync, for 10 us). Warp w counts its routes into cnt[w][e]; the per-expert
// exclusive prefix over the warps plus the expert offset turns cnt into bases; the warps walk
// their routes again and assign stable slots. Same results as the three-kernel path, one launch
// instead of three (the decode and Mixtral-prefill route counts).
constexpr int kSmallUnits = 32;
template <int IT>
__global__ void __launch_bounds__(kSmallUnits * 32)
map_small_kernel(const int32_t *__restrict__ te, int64_t R, int32_t E,
                 int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                 int32_t *__restrict__ sparse_rows, int32_t *__restrict__ sorted_rows,
                 unsigned *status) {
    __shared__ int32_t cnt[kSmallUnits][kMaxE];
    __shared__ int32_t eoff[kMaxE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    for (int e = lane; e < E; e += 32) cnt[warp][e] = 0;
    __syncwarp();
    const int64_t base = (int64_t)warp * (32 * IT);
    // all of this lane's routes at once: IT independent loads instead of a dependent chain
    int ev[IT];
    bool bad = false;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
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
    // one block, latency-bound: warp-aggregated counting with __match_any_sync measured faster
    // here than shared atomics or ballots (the grid path's choices)
#pragma unroll
    for (int it = 0; it < IT; ++it) {
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
        for (int w = 0; w < nw; ++w) {
            const int32_t c = cnt[w][e];
            cnt[w][e] = run;
            run += c;
        }
        eoff[e] = run;
    }
    __syncthreads();
    // expert offsets: exclusive prefix of the totals, 32 experts at a time by warp 0
    if (warp == 0) {
        int32_t carry = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int32_t c = e < E ? eoff[e] : 0;
            int32_t incl = c;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int32_t v = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += v;
            }
            if (e < E) {
                counts[e] = c;
                offsets[e] = carry + incl - c;
                eoff[e] = carry + incl - c;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) offsets[E] = carry;
    }
    __syncthreads();
    for (int e = lane; e < E; e += 32) cnt[warp][e] += eoff[e];
    __syncwarp();
    const unsigned lower = (1u << lane) - 1u;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
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
            if (slot >= 0 && dev::debug_in_range(slot, R, status)) sorted_rows[slot] = (int32_t)i;
        }
    }
}

}  // namespace

namespace {

constexpr int kMinBlocks = 148;  // one block per SM of a B200

// 32-route steps per warp unit of the grid path: 16 once that gives kMinBlocks blocks, else the
// largest of 8, 4, 2 that does, else 1.
int grid_iters(int64_t R) {
    for (int it = kIters; it > 1; it >>= 1) {
        const int64_t br = (int64_t)kWarpsPerBlock * 32 * it;
        if ((R + br - 1) / br >= kMinBlocks) return it;
    }
    return 1;
}

int64_t grid_blocks(int64_t R) {
    const int64_t br = (int64_t)kWarpsPerBlock * 32 * grid_iters(R);
    return (R + br - 1) / br;
}

template <int IT>
void launch_grid(const int32_t *te, int64_t R, int32_t E, int64_t nblk, int32_t *bcount,
                 int32_t *totals, int32_t *counts, int32_t *offsets, int32_t *sparse_rows,
                 int32_t *sorted_rows, unsigned *status, cudaStream_t s) {
    map_count_kernel<IT><<<(unsigned)nblk, kWarpsPerBlock * 32, 0, s>>>(te, R, E, nblk, bcount,
                                                                         status);
    if (nblk > kScanRowsFrom)
        map_scan_rows_kernel<<<(unsigned)E, kScanThreads, 0, s>>>(bcount, nblk, totals);
    else
        map_scan_kernel<<<(unsigned)E, kScanThreads, 0, s>>>(bcount, nblk, totals);
    if (E <= 8 * IT) {
        // the largest table (E = 128 at 16 routes a lane) needs more than the default 48 KB of
        // dynamic shared memory; a failure here surfaces as the launch's error
        static std::once_flag once;
        std::call_once(once, [] {
            cudaFuncSetAttribute(map_assign_lane_kernel<IT>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)AssignSmem<IT>::bytes(8 * IT));
        });
        map_assign_lane_kernel<IT>
            <<<(unsigned)nblk, kWarpsPerBlock * 32, AssignSmem<IT>::bytes(E), s>>>(
                te, R, E, nblk, bcount, totals, counts, offsets, sparse_rows, sorted_rows, status);
        return;
    }
    map_assign_warp_kernel<IT><<<(unsigned)nblk, kWarpsPerBlock * 32, 0, s>>>(
        te, R, E, nblk, bcount, totals, counts, offsets, sparse_rows, sorted_rows, status);
}

}  // namespace

// (blocks + 1) x E words; blocks <= max(ceil(R / 4096), 294).
size_t map_scratch_bytes(int64_t R, int32_t E) {
    const int64_t nblk = grid_blocks(R);
    return (size_t)((nblk > 0 ? nblk : 1) + 1) * (size_t)E * sizeof(int32_t);
}

int launch_sparse_map(const int32_t *te, int64_t R, int32_t E, int32_t *counts, int32_t *offsets,
                      int32_t *sparse_rows, int32_t *sorted_rows, int32_t *scratch,
                      unsigned *status, cudaStream_t s, int *n_launch) {
    const int64_t units = (R + kUnit - 1) / kUnit;
    if (units <= kSmallUnits) {
        // steps per warp: the fewest that keep the warps at or below 32
        int it = 1;
        while (it < kIters && (R + 32 * it - 1) / (32 * it) > kSmallUnits) it *= 2;
        const int warps = (int)std::max<int64_t>(1, (R + 32 * it - 1) / (32 * it));
        auto k = map_small_kernel<16>;
        switch (it) {
            case 1: k = map_small_kernel<1>; break;
            case 2: k = map_small_kernel<2>; break;
            case 4: k = map_small_kernel<4>; break;
            case 8: k = map_small_kernel<8>; break;
            default: break;
        }
        k<<<1, warps * 32, 0, s>>>(te, R, E, counts, offsets, sparse_rows, sorted_rows, status);
        if (n_launch) *n_launch += 1;
        return 0;
    }
    // scratch: block counts / bases [E][nblk], then the expert totals [E]
    const int64_t nblk = grid_blocks(R);
    int32_t *bcount = scratch;
    int32_t *totals = scratch + (int64_t)E * nblk;
    switch (grid_iters(R)) {
        case 16:
            launch_grid<16>(te, R, E, nblk, bcount, totals, counts, offsets, sparse_rows,
                            sorted_rows, status, s);
            break;
        case 8:
            launch_grid<8>(te, R, E, nblk, bcount, totals, counts, offsets, sparse_rows,
                           sorted_rows, status, s);
            break;
        case 4:
            launch_grid<4>(te, R, E, nblk, bcount, totals, counts, offsets, sparse_rows,
                           sorted_rows, status, s);
            break;
        case 2:
            launch_grid<2>(te, R, E, nblk, bcount, totals, counts, offsets, sparse_rows,
                           sorted_rows, status, s);
            break;
        default:
            launch_grid<1>(te, R, E, nblk, bcount, totals, counts, offsets, sparse_rows,
                           sorted_rows, status, s);
            break;
    }
    if (n_launch) *n_launch += 3;
    return 0;
}

}  // namespace moe
