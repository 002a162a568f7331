// kernel_combine.cuh -- split-KV combine (log-sum-exp merge of partials).
//
// For a sequence whose KV tiles were cut across k > 1 partitions, partition
// pieces left (O_s / l_s, lse_s) in fp32.  The merged result is
//     lse = ln sum_s exp(lse_s),      out = sum_s exp(lse_s - lse) * (O_s / l_s)
// which is exactly the softmax over the union of the pieces' keys.  The pages
// do not describe splitting; this is the standard identity for merging
// softmax-normalised partial results.  Sequences that were not cut were
// finished by the main kernel and are skipped; empty sequences (L = 0) are
// written here as out = 0, lse = -inf.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "schedule.cuh"

namespace mla {

struct CombineArgs {
    const int32_t* seqlens;
    int B;
    int R;
    int L_max;
    int P;
    __nv_bfloat16* out;
    float* lse;
    const float* part_o;
    const float* part_lse;
};

constexpr int kCombineThreads = 128;
constexpr int kCombineRowsPerCta = 16;

__global__ void __launch_bounds__(kCombineThreads)
    mla_decode_combine_kernel(const CombineArgs args) {
    __shared__ long long red_acc[kCombineThreads / 32];
    __shared__ long long red_tot[kCombineThreads / 32];
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // flat tile offset of sequence b, and the total
    long long acc = 0, tot = 0;
    for (int i = threadIdx.x; i < args.B; i += kCombineThreads) {
        const long long n = num_tiles(clamp_len(args.seqlens[i], args.L_max, nullptr));
        tot += n;
        if (i < b) acc += n;
    }
    acc = warp_sum_ll(acc);
    tot = warp_sum_ll(tot);
    if (lane == 0) {
        red_acc[warp] = acc;
        red_tot[warp] = tot;
    }
    __syncthreads();
    acc = 0;
    tot = 0;
#pragma unroll
    for (int w = 0; w < kCombineThreads / 32; ++w) {
        acc += red_acc[w];
        tot += red_tot[w];
    }
    const int L = clamp_len(args.seqlens[b], args.L_max, nullptr);
    const long long n = num_tiles(L);
    const int row_lo = blockIdx.y * kCombineRowsPerCta;
    const int row_hi = min(args.R, row_lo + kCombineRowsPerCta);

    if (n == 0) {
        for (int r = row_lo + warp; r < row_hi; r += kCombineThreads / 32) {
            const size_t orow = static_cast<size_t>(b) * args.R + r;
            for (int e = lane; e < kDv; e += 32) args.out[orow * kDv + e] = __float2bfloat16_rn(0.f);
            if (lane == 0) args.lse[orow] = -INFINITY;
        }
        return;
    }
    const long long T = (tot + args.P - 1) / args.P;
    const int p0 = static_cast<int>(acc / T);
    const int p1 = static_cast<int>((acc + n - 1) / T);
    if (p0 == p1) return;  // finished by the main kernel
    const int k = p1 - p0 + 1;

    for (int r = row_lo + warp; r < row_hi; r += kCombineThreads / 32) {
        // pass 1: merged lse
        float m = -INFINITY;
        for (int i = 0; i < k; ++i) {
            const int slot = (i == 0) ? 2 * p0 + 1 : 2 * (p0 + i);
            m = fmaxf(m, args.part_lse[static_cast<size_t>(slot) * args.R + r]);
        }
        float s = 0.f;
        for (int i = 0; i < k; ++i) {
            const int slot = (i == 0) ? 2 * p0 + 1 : 2 * (p0 + i);
            s += expf(args.part_lse[static_cast<size_t>(slot) * args.R + r] - m);
        }
        const float lse_all = m + logf(s);
        // pass 2: weighted sum, 16 columns per lane (4 x float4)
        float acc_o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc_o[e] = 0.f;
        for (int i = 0; i < k; ++i) {
            const int slot = (i == 0) ? 2 * p0 + 1 : 2 * (p0 + i);
            const size_t prow = static_cast<size_t>(slot) * args.R + r;
            const float w = expf(args.part_lse[prow] - lse_all);
            const float4* src = reinterpret_cast<const float4*>(args.part_o + prow * kDv);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float4 x = src[v * 32 + lane];
                acc_o[4 * v + 0] += w * x.x;
                acc_o[4 * v + 1] += w * x.y;
                acc_o[4 * v + 2] += w * x.z;
                acc_o[4 * v + 3] += w * x.w;
            }
        }
        const size_t orow = static_cast<size_t>(b) * args.R + r;
        __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(args.out + orow * kDv);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int e0 = (v * 32 + lane) * 4;  // column of acc_o[4v]
            dst[e0 / 2] = __floats2bfloat162_rn(acc_o[4 * v + 0], acc_o[4 * v + 1]);
            dst[e0 / 2 + 1] = __floats2bfloat162_rn(acc_o[4 * v + 2], acc_o[4 * v + 3]);
        }
        if (lane == 0) args.lse[orow] = lse_all;
    }
}

}  // namespace mla
