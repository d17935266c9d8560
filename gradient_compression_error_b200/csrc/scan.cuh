// scan.cuh -- warp / block prefix sums, the warp bit transpose and the
// radix-bin crossing search.
#pragma once

#include <cstdint>

namespace gce {

constexpr unsigned kFull = 0xFFFFFFFFu;

template <class T>
__device__ __forceinline__ T warp_inclusive_scan(T x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        T y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

template <class T>
__device__ __forceinline__ T warp_sum(T x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    return x;
}

// 32 x 32 bit transpose over a warp: lane r holds row r (bit c = entry (r, c))
// on entry and column r (bit c = entry (c, r)) on return.  Five rounds, each
// swapping the off-diagonal blocks of half the size with the partner lane.
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 16; j >= 1; j >>= 1) {
        const uint32_t m = j == 16 ? 0x0000FFFFu
                         : j == 8  ? 0x00FF00FFu
                         : j == 4  ? 0x0F0F0F0Fu
                         : j == 2  ? 0x33333333u
                                   : 0x55555555u;  // bits whose index has bit j clear
        const uint32_t y = __shfl_xor_sync(kFull, x, j);
        x = (lane & j) ? ((x & ~m) | ((y >> j) & m)) : ((x & m) | ((y << j) & ~m));
    }
    return x;
}

// Exclusive prefix sum over the block (blockDim.x a multiple of 32, <= 1024).
// s_warp: 33 ints of shared scratch.  Returns the thread's exclusive prefix;
// *total receives the block total.  Contains __syncthreads (call uniformly).
__device__ __forceinline__ int block_exclusive_scan(int x, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = warp_inclusive_scan(x);
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = lane < nw ? s_warp[lane] : 0;
        int vi = warp_inclusive_scan(v);
        if (lane < nw) s_warp[lane] = vi - v;
        if (lane == 31) s_warp[32] = vi;  // lane 31 holds the block total
    }
    __syncthreads();
    int res = s_warp[warp] + incl - x;
    *total = s_warp[32];
    __syncthreads();
    return res;
}

// Sum of lane l's run of `per` bins h[l*per .. l*per + per), a power of two.
// Lane l starts its run at a different bin than its neighbours, so the 32
// reads of each step fall in 32 banks when per is a multiple of 32.
__device__ __forceinline__ int64_t warp_run_sum(const int32_t* h, int per) {
    const int lane = threadIdx.x & 31;
    int64_t mine = 0;
    for (int i = 0; i < per; ++i) mine += h[lane * per + ((i + lane) & (per - 1))];
    return mine;
}

// Run by one full warp.  h: nb bins in shared memory, nb a power of two >= 32.
// Finds the bin b with above(b) < target <= above(b) + h[b], where above(b)
// is the sum of all bins above b (the crossing of the count taken from the
// top).  Returns -1 when the total is below target.  *above_out = above(b).
// The run of the lane holding the crossing is then split over the warp, q
// bins a lane, and only the q bins of the lane holding it are scanned in turn.
__device__ __forceinline__ int warp_find_from_top(const int32_t* h, int nb, int64_t target,
                                                  int64_t* above_out) {
    const int lane = threadIdx.x & 31;
    const int per = nb >> 5;
    const int64_t mine = warp_run_sum(h, per);
    // inclusive suffix sum over lanes (this lane and every higher one)
    int64_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int64_t y = __shfl_down_sync(kFull, incl, o);
        if (lane + o < 32) incl += y;
    }
    const int64_t excl = incl - mine;
    const unsigned ball = __ballot_sync(kFull, excl < target && target <= incl);
    if (ball == 0) {
        *above_out = __shfl_sync(kFull, incl, 0);
        return -1;
    }
    const int src = __ffs(ball) - 1;
    const int64_t above_src = __shfl_sync(kFull, excl, src);
    // lane j takes the j-th group of q bins from the top of src's run
    const int q = per >= 32 ? per >> 5 : 1;
    const int top = src * per + per - lane * q;  // one past this lane's group
    int64_t sub = 0;
    if (lane * q < per)
        for (int i = 1; i <= q; ++i) sub += h[top - i];
    const int64_t pin = warp_inclusive_scan(sub);  // groups at or above this lane's
    const int64_t t2 = target - above_src;
    const unsigned b2 = __ballot_sync(kFull, pin - sub < t2 && t2 <= pin);
    const int s2 = __ffs(b2) - 1;  // b2 is never empty: src's run holds the crossing
    int res = -1;
    int64_t above = 0;
    if (lane == s2) {
        int64_t acc = above_src + pin - sub;
        for (int b = top - 1; b >= top - q; --b) {
            if (acc + h[b] >= target) {
                res = b;
                above = acc;
                break;
            }
            acc += h[b];
        }
    }
    res = __shfl_sync(kFull, res, s2);
    above = __shfl_sync(kFull, above, s2);
    *above_out = above;
    return res;
}

// As warp_find_from_top, counting from the bottom: returns b with
// below(b) < target <= below(b) + h[b]; *below_out = below(b).
__device__ __forceinline__ int warp_find_from_bottom(const int32_t* h, int nb, int64_t target,
                                                     int64_t* below_out) {
    const int lane = threadIdx.x & 31;
    const int per = nb >> 5;
    const int64_t mine = warp_run_sum(h, per);
    const int64_t incl = warp_inclusive_scan(mine);
    const int64_t excl = incl - mine;
    const unsigned ball = __ballot_sync(kFull, excl < target && target <= incl);
    if (ball == 0) {
        *below_out = __shfl_sync(kFull, incl, 31);
        return -1;
    }
    const int src = __ffs(ball) - 1;
    const int64_t below_src = __shfl_sync(kFull, excl, src);
    // lane j takes the j-th group of q bins from the bottom of src's run
    const int q = per >= 32 ? per >> 5 : 1;
    const int bot = src * per + lane * q;  // this lane's first bin
    int64_t sub = 0;
    if (lane * q < per)
        for (int i = 0; i < q; ++i) sub += h[bot + i];
    const int64_t pin = warp_inclusive_scan(sub);
    const int64_t t2 = target - below_src;
    const unsigned b2 = __ballot_sync(kFull, pin - sub < t2 && t2 <= pin);
    const int s2 = __ffs(b2) - 1;  // never empty: src's run holds the crossing
    int res = -1;
    int64_t below = 0;
    if (lane == s2) {
        int64_t acc = below_src + pin - sub;
        for (int b = bot; b < bot + q; ++b) {
            if (acc + h[b] >= target) {
                res = b;
                below = acc;
                break;
            }
            acc += h[b];
        }
    }
    res = __shfl_sync(kFull, res, s2);
    below = __shfl_sync(kFull, below, s2);
    *below_out = below;
    return res;
}

}  // namespace gce
