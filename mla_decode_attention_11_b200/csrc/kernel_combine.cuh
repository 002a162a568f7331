// kernel_combine.cuh -- split-KV combine (log-sum-exp merge of partials).
//
// For a sequence whose KV tiles were cut across k > 1 partitions, partition
// pieces left (O_s / l_s, lse_s) in fp32.  The merged result is
//     lse = ln sum_s exp(lse_s),      out = sum_s exp(lse_s - lse) * (O_s / l_s)
// which is exactly the softmax over the union of the pieces' keys.  A
// per-head attention sink (one more softmax term without a value) enters the
// merged lse only, once per row.  The pages
// do not describe splitting; this is the standard identity for merging
// softmax-normalised partial results.  Sequences that were not cut were
// finished by the main kernel and are skipped; empty sequences (L = 0) are
// written here as out = 0, lse = -inf (or the head's sink logit).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
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
    const float* sinks;  // [H] per-head attention-sink logits (natural-log units), or null
    int H;
    int split_tiles;     // 0: balanced schedule; > 0: batch-invariant chunks of this many tiles
};

// Grid (B, Y): CTA (b, y) owns sequence b's query rows [y*RY, (y+1)*RY) with
// RY = ceil(R / Y); its 8 warps take one row each at a time.  Warp 0 reads the
// lengths once (schedule and b's unit offset in one pass), so a sequence that
// was not cut costs its CTAs one scan and nothing else; Y is chosen by the
// host so that about two CTAs per SM share the merging of cut sequences.
// Within a row the kernel is bound by the latency of the partials it reads, so
// each lane keeps up to 4 partials x 4 float4 in flight, requested before the
// merged lse is known, instead of walking the partials one after another.
constexpr int kCombineThreads = 256;
constexpr int kCombineWarps = kCombineThreads / 32;

// CTAs per sequence along y: enough to give about two CTAs per SM when many
// rows must be merged, never more than one per 8 rows.
inline int combine_grid_y(int B, int R, int num_sms) {
    const int max_y = (R + kCombineWarps - 1) / kCombineWarps;
    int y = (2 * num_sms) / B;
    if (y < 1) y = 1;
    return y < max_y ? y : max_y;
}

// DV: value width (512 for MLA, 128 for MHA); a lane owns DV / 128 float4 columns.
template <int DV = kDv>
__global__ void __launch_bounds__(kCombineThreads, 2)
    mla_decode_combine_kernel(const CombineArgs args) {
    static_assert(DV == 512 || DV == 128, "value width");
    constexpr int NV4 = DV / 128;  // float4 columns per lane
    __shared__ int s_split;
    __shared__ long long s_acc, s_tot;
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // the schedule the main kernel used for these lengths, its unit count and
    // the flat unit offset of sequence b (units: tiles, or S-tile chunks)
    if (warp == 0) {
        const ScheduleScan sc = schedule_scan_warp(args.seqlens, args.B, args.L_max, args.P, args.split_tiles, b);
        if (lane == 0) {
            s_split = sc.S;
            s_acc = sc.acc_at;
            s_tot = sc.units;
        }
    }
    __syncthreads();
    // launched as a programmatic dependent of the main kernel: the scan above
    // reads only the lengths; partials and outputs wait for the main grid
    ptx::wait_prior_grid();
    const int S = s_split;
    const long long acc = s_acc, tot = s_tot;
    const int rows_per = (args.R + static_cast<int>(gridDim.y) - 1) / static_cast<int>(gridDim.y);
    const int r_lo = static_cast<int>(blockIdx.y) * rows_per;
    const int r_hi = r_lo + rows_per < args.R ? r_lo + rows_per : args.R;
    const int L = clamp_len(__ldg(args.seqlens + b), args.L_max, nullptr);
    const long long n = num_units(L, S);
    if (n == 0) {
        for (int r = r_lo + warp; r < r_hi; r += kCombineWarps) {
            const size_t orow = static_cast<size_t>(b) * args.R + r;
            // a per-head sink is one more softmax term without a value (-inf: none)
            const float sink = args.sinks ? args.sinks[r % args.H] : -INFINITY;
            uint4* dst = reinterpret_cast<uint4*>(args.out + orow * DV);  // DV / 8 x 16 bytes
            for (int i = lane; i < DV / 8; i += 32) dst[i] = make_uint4(0u, 0u, 0u, 0u);
            if (lane == 0) args.lse[orow] = sink;  // nothing to attend to: the sink alone
        }
        return;
    }
    int k, p0 = 0;
    if (S > 0) {
        // chunk schedule: chunk i of b is in slot acc + i
        if (n == 1) return;  // one chunk: finished by the main kernel
        k = static_cast<int>(n);
    } else {
        const long long T = (tot + args.P - 1) / args.P;
        p0 = static_cast<int>(acc / T);
        const int p1 = static_cast<int>((acc + n - 1) / T);
        if (p0 == p1) return;  // finished by the main kernel
        k = p1 - p0 + 1;
    }
    // slot of the i-th piece: the first partition's piece continues after it
    // (2 p0 + 1), every later piece started before its partition (2 p)
    auto slot_of = [&](int i) {
        if (S > 0) return static_cast<int>(acc) + i;
        return (i == 0) ? 2 * p0 + 1 : 2 * (p0 + i);
    };

    for (int r = r_lo + warp; r < r_hi; r += kCombineWarps) {
        const size_t orow = static_cast<size_t>(b) * args.R + r;
        const float sink = args.sinks ? args.sinks[r % args.H] : -INFINITY;
        auto prow_of = [&](int i) { return static_cast<size_t>(slot_of(i)) * args.R + r; };
        // the first (up to) 4 partial rows are requested before the lse values
        // are reduced, so a row cut into at most 4 pieces costs one round trip
        float4 x[4][NV4];
        auto load_batch = [&](int i0) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (i0 + j < k) {
                    const float4* src = reinterpret_cast<const float4*>(args.part_o + prow_of(i0 + j) * DV);
#pragma unroll
                    for (int v = 0; v < NV4; ++v) x[j][v] = __ldcs(src + lane + 32 * v);
                }
            }
        };
        load_batch(0);
        // merged lse: lane i holds piece i (pieces beyond 32 folded in by a loop)
        const float my_l = lane < k ? args.part_lse[prow_of(lane)] : -INFINITY;
        float m = my_l;
        for (int i = lane + 32; i < k; i += 32) m = fmaxf(m, args.part_lse[prow_of(i)]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        m = fmaxf(m, sink);
        const float my_e = lane < k ? expf(my_l - m) : 0.f;
        float sum = my_e;
        for (int i = lane + 32; i < k; i += 32) sum += expf(args.part_lse[prow_of(i)] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        sum += expf(sink - m);
        const float lse_all = m + logf(sum);
        const float inv = 1.f / sum;
        const float my_w = my_e * inv;  // weight of piece `lane`: exp(lse_lane - lse)

        // out = sum_i exp(lse_i - lse) * (O_i / l_i); lane owns float4 columns lane + 32 v
        float4 acc_o[NV4];
#pragma unroll
        for (int v = 0; v < NV4; ++v) acc_o[v] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i0 = 0; i0 < k; i0 += 4) {
            if (i0 > 0) load_batch(i0);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = i0 + j;
                if (i < k) {
                    const float w = i < 32 ? __shfl_sync(0xffffffffu, my_w, i)
                                           : expf(args.part_lse[prow_of(i)] - m) * inv;
#pragma unroll
                    for (int v = 0; v < NV4; ++v) {
                        acc_o[v].x += w * x[j][v].x;
                        acc_o[v].y += w * x[j][v].y;
                        acc_o[v].z += w * x[j][v].z;
                        acc_o[v].w += w * x[j][v].w;
                    }
                }
            }
        }
        __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(args.out + orow * DV);
#pragma unroll
        for (int v = 0; v < NV4; ++v) {
            const int e0 = (lane + 32 * v) * 4;  // first column of acc_o[v]
            const __nv_bfloat162 lo = __floats2bfloat162_rn(acc_o[v].x, acc_o[v].y);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(acc_o[v].z, acc_o[v].w);
            uint2 pk;
            pk.x = *reinterpret_cast<const uint32_t*>(&lo);
            pk.y = *reinterpret_cast<const uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(dst + e0 / 2) = pk;
        }
        if (lane == 0) args.lse[orow] = lse_all;
    }
}

}  // namespace mla
