// kernel_transposed.cuh -- MLA decode main kernel, "transposed" orientation.
//
// One CTA handles G query rows (token, head pairs) of one sequence over one
// contiguous range of its KV tiles.  Per 128-row KV tile:
//
//   S^T[128 kv, G] = K_tile[128, 576] . Q_g^T       tcgen05.mma M=128 N=G K=576
//   softmax over the kv axis (TMEM lanes) in fp32, base 2, lazily rescaled
//   O^T[512, G]   += V_tile^T[512, 128] . P^T        4 x tcgen05.mma M=128 N=G K=128
//
// This is the pages' two-GEMM dataflow ("TileLang: Bridging Programmability and
// Performance in Modern Neural Kernels", papernotes.org, section "一个完整示例：
// FlashMLA 的两阶段优化": Q and the KV tile staged in shared memory, S produced
// by the first GEMM, cast, and fed to the second) re-laid out for sm_100a: the
// accumulators live in tensor memory, the kv rows sit on the 128 TMEM lanes so
// that a small number of query rows (G = 16 or 32) still fills an M=128 MMA,
// and V is read in place as the first 512 columns of the very tile K came in
// (no second load).  The pipeline is warp specialised ("TileLang 完整解析",
// section "三大核心優化機制": a TMA producer warp and consumer warps joined by
// mbarriers), with one warp issuing all tcgen05 MMAs.
//
// Warp roles (192 threads; 320 with an FP8 cache):
//   warps 0-3  softmax + epilogue (thread = TMEM lane = kv row / dv row)
//   warp 4     TMA producer (one elected lane)
//   warp 5     TMEM allocator + MMA issuer (one elected lane)
//   warps 6-9  FP8 cache only (6-7 at G = 32): widen staged E4M3 chunks to f16
//              operands (thread = kv row), and Q from bf16 to f16 once per piece
//
// Shared memory (1024-byte aligned regions, 128-byte swizzle for TMA data):
//   pair ring  NP x 32 KB: a [128 kv x 128 col] block = dv chunks 2p, 2p+1
//   rope ring  NR x 16 KB: the [128 kv x 64] rope chunk (columns 512..575)
//   Q          9 x [G x 64] chunks, loaded once per piece
//   P^T        [128 kv x G] bf16 (f16 with an FP8 cache), MN-major (q contiguous),
//              32/64-byte swizzle
//   FP8 ring   NF x 8 KB: [128 kv x 64] E4M3 codes, 64-byte swizzle (FP8 cache only)
// Every pipeline wait is bounded (%globaltimer); on expiry the CTA records
// kStatusTimeout, drains its own TMA loads and MMAs, frees TMEM and returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "ptx.cuh"
#include "schedule.cuh"

namespace mla {

struct MainArgs {
    const int32_t* seqlens;
    int B;
    int R;            // query rows per sequence (Sq * H)
    int L_max;
    int P;            // partitions
    int NG;           // query-row groups per partition (CTAs sharing a partition)
    float scale_log2; // softmax_scale * log2(e)
    __nv_bfloat16* out;
    float* lse;
    float* part_o;    // [2P, R, 512]
    float* part_lse;  // [2P, R]
    uint32_t* status;
    unsigned long long timeout_ns;
    int stall_unit;   // test hook: skip this TMA unit in CTA 0 (-1 = off)
    int prefetch_tiles;  // KV tiles to prefetch into L2 ahead of the loads (0 = off)
    const float* sinks;  // [H] per-head attention-sink logits (natural-log units), or null
    int H;               // heads: query row r of a sequence belongs to head r % H
    int split_tiles;     // 0: balanced schedule; > 0: batch-invariant chunks of this many tiles
    int Sq;              // query tokens per sequence
    int Hkv;             // MHA: kv heads (query head h reads kv head h / (H / Hkv)); MLA: 1
    float o_scale;       // factor on every output row: the FP8 cache's kv_scale, else 1
    const __nv_bfloat16* q;  // [B*R, 576] query rows (read directly by the FP8-operand kernel)
};

// The two attention shapes the transposed kernel serves.
struct MlaShape {  // latent cache: keys are 576-wide kv rows, values their first 512 columns
    static constexpr bool kMha = false;
    static constexpr bool kFp8 = false;
    static constexpr int kQKChunks = 9;  // 64-column chunks of a key (chunk 8 = rope)
    static constexpr int kDvBlocks = 4;  // 128-wide blocks of a value row
    static constexpr int kDv = 512;
};
struct MhaShape {  // multi-head attention: separate K and V tensors, 128 wide, grouped kv heads
    static constexpr bool kMha = true;
    static constexpr bool kFp8 = false;
    static constexpr int kQKChunks = 2;
    static constexpr int kDvBlocks = 1;
    static constexpr int kDv = 128;
};
// The latent cache stored as E4M3 codes with one dequantization scale: each
// 64-column chunk is staged as 8 KB of codes, widened to f16 in shared memory
// by the converter warps (every E4M3 value, divided by 2^8, is exact in f16),
// and the MMAs run kind::f16 on f16 operands (Q is narrowed from bf16 to f16
// once per piece, P^T is written as f16).  kv_scale * 2^8 enters the score
// scale and o_scale.
struct MlaFp8Shape {
    static constexpr bool kMha = false;
    static constexpr bool kFp8 = true;
    static constexpr int kQKChunks = 9;
    static constexpr int kDvBlocks = 4;
    static constexpr int kDv = 512;
};

// Folds a per-head attention sink into a finished row.  (m, l) are the row's
// base-2 reference max and sum over its keys, s2 the sink in base-2 units
// (-inf: no sink).  The sink is one more softmax term without a value:
// afterwards m = max(m, s2) and l = l 2^(m_old - m) + 2^(s2 - m), and the
// returned factor 2^(m_old - m) rescales the row's O before it is divided
// by the new l.
__device__ __forceinline__ float fold_sink(float& m, float& l, float s2) {
    const float mn = fmaxf(m, s2);
    const float c = exp2f(m - mn);
    l = l * c + exp2f(s2 - mn);
    m = mn;
    return c;
}

constexpr float kLog2e = 1.4426950408889634074f;

// FP8 cache at G = 16: operand pair slots and 8-KB staging slots (5 + 3 fill
// the shared memory; a pair slot can be traded for four staging slots)
#ifndef MLA_FP8_NP16
#define MLA_FP8_NP16 5
#endif
#ifndef MLA_FP8_NF16
#define MLA_FP8_NF16 3
#endif

template <int G, class SH = MlaShape>
struct TransposedCfg {
    static_assert(G == 16 || G == 32, "query rows per CTA");
    // FP8 cache: + 4 converter warps (2 at G = 32, whose softmax needs the
    // registers of a 256-thread block)
    static constexpr int kConvThreads = SH::kFp8 ? ((G == 16) ? 128 : 64) : 0;
    static constexpr int kThreads = 192 + kConvThreads;
    // pair slots [128 kv x 128 col]: an MLA tile needs 4 (+ a rope slot), an MHA
    // tile 2 (its K and its V)
    static constexpr int NP = SH::kMha ? 6 : SH::kFp8 ? ((G == 16) ? MLA_FP8_NP16 : 4) : ((G == 16) ? 5 : 4);
    static constexpr int NR = (SH::kMha || SH::kFp8) ? 1 : 2;  // rope slots (unused by MHA)
    static constexpr int NF = SH::kFp8 ? ((G == 16) ? MLA_FP8_NF16 : 4) : 0;  // FP8 staging slots
    static constexpr int kPairBytes = kTileKV * 128 * 2;     // 32 KB
    static constexpr int kChunkBytes = kTileKV * 128;        // 16 KB
    static constexpr int kF8Bytes = kTileKV * kChunk;        // 8 KB: one chunk of E4M3 codes
    static constexpr int kQChunkBytes = G * 128;
    static constexpr int kPTBytes = kTileKV * G * 2;
    static constexpr int OFF_PAIR = 0;
    static constexpr int OFF_ROPE = OFF_PAIR + NP * kPairBytes;
    static constexpr int OFF_Q = OFF_ROPE + NR * kChunkBytes;
    static constexpr int OFF_PT = OFF_Q + SH::kQKChunks * kQChunkBytes;
    static constexpr int OFF_F8 = OFF_PT + kPTBytes;
    static constexpr int OFF_RED = OFF_F8 + NF * kF8Bytes;          // floats: [2][4][G] max, [4][G] sums
    static constexpr int kRedFloats = 12 * G;
    static constexpr int OFF_BAR = OFF_RED + kRedFloats * 4;
    // barriers: q_full, q_empty, s_full, p_full, pv_done, drain, group_sync, pair_full[NP],
    //           pair_empty[NP], rope_full[NR], rope_empty[NR], f8_full[NF], f8_empty[NF], q_ready
    static constexpr int kNumBars = 7 + 2 * NP + 2 * NR + 2 * NF + (SH::kFp8 ? 1 : 0);
    static constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
    static constexpr int kSmemBytes = OFF_MISC + 64 + 1024;  // + slack to align the base to 1024
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    // TMEM: O^T blocks at columns [0, kDvBlocks G), S^T after them
    static constexpr int kCols = (SH::kDvBlocks + 1) * G;
    static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128 : 256;
    static constexpr uint32_t kColS = SH::kDvBlocks * G;
    // P^T swizzle: one row of G bf16 = 2G bytes (32 or 64)
    static constexpr ptx::Swizzle kPTSwz = (G == 16) ? ptx::Swizzle::B32 : ptx::Swizzle::B64;
    static constexpr uint32_t kPTAtom = 8 * 2 * G;  // 8 rows x row bytes
    static constexpr uint32_t kIdescS =
        SH::kFp8 ? ptx::make_idesc_f16(128, G, 0, 0) : ptx::make_idesc_bf16(128, G, 0, 0);
    static constexpr uint32_t kIdescPV =
        SH::kFp8 ? ptx::make_idesc_f16(128, G, 1, 1) : ptx::make_idesc_bf16(128, G, 1, 1);
};

// Byte offset of 16-byte unit u of row r in a swizzled region whose rows are
// `row_bytes` long (32, 64 or 128) -- the XOR pattern TMA and the UMMA
// descriptors use: unit index ^= (address bits [7, 7+log2(row_bytes/16))).
__device__ __forceinline__ uint32_t swz_offset(uint32_t r, uint32_t u, uint32_t row_bytes) {
    const uint32_t addr = r * row_bytes + u * 16;
    const uint32_t mask = (row_bytes / 16) - 1;
    return addr ^ (((addr >> 7) & mask) << 4);
}

// Widening E4M3 codes to f16 values e4m3(code) * 2^-8 (exact; the kernel
// multiplies the 2^8 back into the score scale and the output scale).  Two
// routes, used for alternate words of a chunk because each alone saturates
// its pipe (measured: half and half is ~10% faster than either):
//  - integer ALU: a code s.eeee.mmm placed in an f16 as s.0eeee.mmm0000000 is,
//    bit for bit, the f16 of e4m3(code) * 2^-8 (normals 2^(e-7)(1 + m/8) become
//    2^(e-15)(1 + m/8), subnormals (m/8) 2^-6 become the f16 subnormals
//    (m/8) 2^-14);
//  - the hardware e4m3x2 -> f16x2 conversion, then an exact f16 multiply by 2^-8.
// The cache must hold finite codes: the integer route reads the NaN codes
// S.1111.111 as +-480 * 2^-8.
constexpr float kF8Unscale = 256.f;

// Four codes (byte k = column k) -> f16 pairs (columns 0, 1) and (2, 3), each
// value e4m3(code) * 2^-8.
__device__ __forceinline__ void e4m3x4_to_f16x4_div256(uint32_t codes, uint32_t& lo, uint32_t& hi) {
    const uint32_t w0 = __byte_perm(codes, 0u, 0x1404u);  // code 1 << 24 | code 0 << 8
    const uint32_t w1 = __byte_perm(codes, 0u, 0x3424u);  // code 3 << 24 | code 2 << 8
    lo = ((w0 & 0x7F007F00u) >> 1) | (w0 & 0x80008000u);
    hi = ((w1 & 0x7F007F00u) >> 1) | (w1 & 0x80008000u);
}

// The same four values through the conversion unit.
__device__ __forceinline__ void e4m3x4_to_f16x4_div256_cvt(uint32_t codes, uint32_t& lo, uint32_t& hi) {
    const __half2 k = __float2half2_rn(0.00390625f);  // 2^-8
    __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(codes & 0xFFFFu), __NV_E4M3);
    __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(codes >> 16), __NV_E4M3);
    const __half2 ha = __hmul2(*reinterpret_cast<const __half2*>(&a), k);
    const __half2 hb = __hmul2(*reinterpret_cast<const __half2*>(&b), k);
    lo = *reinterpret_cast<const uint32_t*>(&ha);
    hi = *reinterpret_cast<const uint32_t*>(&hb);
}

// Eight bf16 -> eight f16 (round to nearest even; exact for |x| in [2^-17, 65504]).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        const __half2 h = __float22half2_rn(f);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Widens kv row r of one staged chunk: 64 E4M3 codes (64-byte rows, 64-byte
// swizzle, as TMA wrote them) -> 64 f16 (each e4m3(code) * 2^-8) in the
// 128-byte-swizzled K-major layout the MMA descriptors read (the layout TMA
// gives a bf16 chunk).
__device__ __forceinline__ void widen_chunk_row(const uint8_t* f8, uint8_t* dst, uint32_t r) {
#pragma unroll
    for (uint32_t u = 0; u < 4; ++u) {
        const uint4 c = *reinterpret_cast<const uint4*>(f8 + swz_offset(r, u, 64));
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (i < 2)
                e4m3x4_to_f16x4_div256_cvt(w[i], o[2 * i], o[2 * i + 1]);
            else
                e4m3x4_to_f16x4_div256(w[i], o[2 * i], o[2 * i + 1]);
        }
        *reinterpret_cast<uint4*>(dst + swz_offset(r, 2 * u, 128)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(dst + swz_offset(r, 2 * u + 1, 128)) = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Warp reduce-scatter: v[0..G) per lane -> on return, every lane holds the
// reduction over the 32 lanes of column col_of_lane(lane) in its return value.
template <int G, bool kMax>
__device__ __forceinline__ float warp_reduce_scatter(const float (&v_in)[G], int lane) {
    constexpr int LOG2G = (G == 16) ? 4 : 5;
    float v[G];
#pragma unroll
    for (int i = 0; i < G; ++i) v[i] = v_in[i];
#pragma unroll
    for (int s = 0; s < LOG2G; ++s) {
        const int h = G >> (s + 1);
        const int mask = 16 >> s;
        const bool upper = (lane & mask) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = upper ? v[i] : v[i + h];
            const float keep = upper ? v[i + h] : v[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, mask);
            v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
#pragma unroll
    for (int m = (16 >> LOG2G); m >= 1; m >>= 1) {
        const float recv = __shfl_xor_sync(0xffffffffu, v[0], m);
        v[0] = kMax ? fmaxf(v[0], recv) : v[0] + recv;
    }
    return v[0];
}

template <int G>
__device__ __forceinline__ int col_of_lane(int lane) {
    return (G == 32) ? lane : (lane >> 1);
}

// MHA (SH = MhaShape): CTA group g is kv head g; its columns j < Sq * (H / Hkv)
// are the query rows (token j / gq, head g gq + j % gq), gq = H / Hkv; the
// remaining columns up to G are padding (zero Q, never stored).  tm_kv is K
// and tm_v is V, both [B, L_max, Hkv, 128].  MLA: group g is query rows
// [g G, g G + G) of the sequence and tm_v is unused.
template <class SH>
__device__ __forceinline__ int group_row(const MainArgs& a, int G, int g, int j) {
    if (!SH::kMha) return g * G + j;
    const int gq = a.H / a.Hkv;
    return (j / gq) * a.H + g * gq + (j % gq);
}

template <int G, class SH = MlaShape>
__global__ void __launch_bounds__(TransposedCfg<G, SH>::kThreads, 1)
    mla_decode_transposed_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                                 const __grid_constant__ CUtensorMap tm_v, const MainArgs args) {
    using C = TransposedCfg<G, SH>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    uint8_t* pair_smem = smem + C::OFF_PAIR;
    uint8_t* rope_smem = smem + C::OFF_ROPE;
    uint8_t* q_smem = smem + C::OFF_Q;
    uint8_t* pt_smem = smem + C::OFF_PT;
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars + 0;
    uint64_t* q_empty = bars + 1;
    uint64_t* s_full = bars + 2;
    uint64_t* p_full = bars + 3;
    uint64_t* pv_done = bars + 4;
    uint64_t* drain = bars + 5;
    uint64_t* group_sync = bars + 6;  // the 128 softmax threads (bounded, unlike bar.sync)
    uint64_t* pair_full = bars + 7;
    uint64_t* pair_empty = pair_full + C::NP;
    uint64_t* rope_full = pair_empty + C::NP;
    uint64_t* rope_empty = rope_full + C::NR;
    uint64_t* f8_full = rope_empty + C::NR;   // FP8 staging slot landed (TMA)
    uint64_t* f8_empty = f8_full + C::NF;     // FP8 staging slot widened (converters)
    uint64_t* q_ready = f8_empty + C::NF;     // FP8: Q narrowed to f16 in place
    uint8_t* f8_smem = smem + C::OFF_F8;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    uint32_t* tmem_base_slot = misc + 0;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    int* b_first_slot = reinterpret_cast<int*>(misc + 2);
    long long* acc_first_slot = reinterpret_cast<long long*>(misc + 4);
    long long* total_slot = reinterpret_cast<long long*>(misc + 6);
    int* split_slot = reinterpret_cast<int*>(misc + 8);  // schedule chunk size of this run (0: balanced)

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int p = blockIdx.x / args.NG;  // partition
    const int g = blockIdx.x % args.NG;  // query-row group within the sequence

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        ptx::mbar_init(q_full, 1);
        ptx::mbar_init(q_empty, 1);
        ptx::mbar_init(s_full, 1);
        ptx::mbar_init(p_full, 128);
        ptx::mbar_init(pv_done, 1);
        ptx::mbar_init(drain, 1);
        ptx::mbar_init(group_sync, 128);
        // FP8: the converter threads fill the operand slots, not TMA
        const uint32_t fill_count = SH::kFp8 ? C::kConvThreads : 1;
        for (int i = 0; i < C::NP; ++i) {
            ptx::mbar_init(pair_full + i, fill_count);
            ptx::mbar_init(pair_empty + i, 1);
        }
        for (int i = 0; i < C::NR; ++i) {
            ptx::mbar_init(rope_full + i, fill_count);
            ptx::mbar_init(rope_empty + i, 1);
        }
        for (int i = 0; i < C::NF; ++i) {
            ptx::mbar_init(f8_full + i, 1);
            ptx::mbar_init(f8_empty + i, C::kConvThreads);
        }
        if (SH::kFp8) ptx::mbar_init(q_ready, C::kConvThreads);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
    }
    if (warp == 5) {
        ptx::tmem_alloc<C::kTmemCols>(tmem_base_slot);
        ptx::tmem_relinquish();
    }
    if (warp == 0) {
        const ScheduleScan sc = schedule_scan_warp(args.seqlens, args.B, args.L_max, args.P, args.split_tiles);
        const int S_eff = sc.S;
        // partition bounds in the flat tile space, and the first sequence
        const long long total = sc.units;
        const long long T = (total + args.P - 1) / args.P;
        const long long start = static_cast<long long>(p) * T;
        int bf;
        long long af;
        locate_warp(args.seqlens, args.B, args.L_max, S_eff, start, &bf, &af);
        if (lane == 0) {
            *b_first_slot = bf;
            *acc_first_slot = af;
            *total_slot = total;
            *split_slot = S_eff;
        }
        // flag out-of-range lengths once (partition 0, group 0 only)
        if (blockIdx.x == 0)
            for (int b = lane; b < args.B; b += 32) clamp_len(args.seqlens[b], args.L_max, args.status);
    }
    if (warp == 4 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_kv);
        if (SH::kMha) ptx::prefetch_tmap(&tm_v);
    }
    if (SH::kMha) {
        // the Q rows past Sq * gq are padding that TMA never writes: make them zero
        for (int i = threadIdx.x; i < SH::kQKChunks * C::kQChunkBytes / 16; i += C::kThreads)
            reinterpret_cast<uint4*>(q_smem)[i] = make_uint4(0u, 0u, 0u, 0u);
        ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;
    // the split-KV combine (launched after this kernel as a programmatic
    // dependent) may start scheduling its CTAs; it waits for this grid's results
    ptx::launch_dependents();

    PieceWalker walker;
    {
        const long long total = *total_slot;
        const long long T = (total + args.P - 1) / args.P;
        walker.seqlens = args.seqlens;
        walker.B = args.B;
        walker.L_max = args.L_max;
        walker.p = p;
        walker.S = *split_slot;
        walker.k = 0;
        walker.start = static_cast<long long>(p) * T;
        walker.end = walker.start + T < total ? walker.start + T : total;
        walker.b = *b_first_slot;
        walker.acc = *acc_first_slot;
    }
    const uint64_t tmo = args.timeout_ns;

    if (warp == 4) {
        // ============================================================ TMA producer
        if (ptx::elect_one()) {
            uint32_t pair_cnt = 0, rope_cnt = 0, piece_cnt = 0, f8_cnt = 0;
            int unit = 0;
            // FP8 cache: L2 prefetch cursor `prefetch_tiles` tiles ahead of the
            // staging loads, across piece boundaries (a tile's 9 chunk boxes,
            // and the next piece's Q rows on entering it).  The staging ring
            // holds few bytes, so without it the loads see HBM latency.
            PieceWalker pf_walker = walker;
            Piece pf_pc{};
            bool pf_live = false, pf_started = false;
            int pf_t = 0;
            auto prefetch_next = [&](bool issue) {
                if (!pf_live) return;
                int r0 = pf_t * kTileKV;
                if (r0 + kTileKV > pf_pc.L) r0 = pf_pc.L - kTileKV;
                if (issue)
                    for (int j = 0; j < kNumChunks; ++j) ptx::tma_prefetch_3d(&tm_kv, j * kChunk, r0, pf_pc.b);
                if (++pf_t == pf_pc.tile_hi) {
                    pf_live = pf_walker.next(pf_pc);
                    if (pf_live) {
                        pf_t = pf_pc.tile_lo;
                        const int qrow = pf_pc.b * args.R + g * G;
                        for (int c = 0; c < kNumChunks; ++c) ptx::tma_prefetch_2d(&tm_q, c * kChunk, qrow);
                    }
                }
            };
            bool ok = true;
            // last armed phase per slot, for the drain on abort
            Piece pc;
            while (ok && walker.next(pc)) {
                // Q rows of this group: flattened [B*R, 576] rows b*R + g*G ...
                if (piece_cnt > 0) ok = ptx::mbar_wait_bounded(q_empty, (piece_cnt - 1) & 1, tmo);
                if (!ok) break;
                if (SH::kMha) {
                    // q viewed as [B][Sq][H][128]: heads g gq .. g gq + gq - 1 of every token
                    const int gq = args.H / args.Hkv;
                    ptx::mbar_arrive_expect_tx(q_full, SH::kQKChunks * args.Sq * gq * 128);
                    if (!(blockIdx.x == 0 && unit == args.stall_unit))
                        for (int c = 0; c < SH::kQKChunks; ++c)
                            ptx::tma_load_4d(q_smem + c * C::kQChunkBytes, &tm_q, q_full, c * kChunk, g * gq, 0, pc.b);
                } else {
                    ptx::mbar_arrive_expect_tx(q_full, kNumChunks * C::kQChunkBytes);
                    const int qrow = pc.b * args.R + g * G;
                    if (!(blockIdx.x == 0 && unit == args.stall_unit))
                        for (int c = 0; c < kNumChunks; ++c)
                            ptx::tma_load_2d(q_smem + c * C::kQChunkBytes, &tm_q, q_full, c * kChunk, qrow);
                }
                ++unit;
                for (int t = pc.tile_lo; t < pc.tile_hi && ok; ++t) {
                    int row0 = t * kTileKV;
                    if (row0 + kTileKV > pc.L) row0 = pc.L - kTileKV;  // end-aligned last tile
                    if (SH::kMha) {
                        // two pair slots: the tile's K rows, then its V rows (kv head g)
                        for (int pp = 0; pp < 2; ++pp) {
                            const uint32_t s = pair_cnt % C::NP;
                            ok = ptx::mbar_wait_bounded(pair_empty + s, ((pair_cnt / C::NP) & 1) ^ 1, tmo);
                            if (!ok) break;
                            ptx::mbar_arrive_expect_tx(pair_full + s, C::kPairBytes);
                            if (!(blockIdx.x == 0 && unit == args.stall_unit)) {
                                uint8_t* dst = pair_smem + s * C::kPairBytes;
                                const CUtensorMap* tm = (pp == 0) ? &tm_kv : &tm_v;
                                ptx::tma_load_4d(dst, tm, pair_full + s, 0, g, row0, pc.b);
                                ptx::tma_load_4d(dst + C::kChunkBytes, tm, pair_full + s, kChunk, g, row0, pc.b);
                            }
                            ++unit;
                            ++pair_cnt;
                        }
                        continue;
                    }
                    if constexpr (SH::kFp8) {
                        if (!pf_started) {
                            pf_started = true;
                            pf_live = args.prefetch_tiles > 0 && pf_walker.next(pf_pc);
                            pf_t = pf_live ? pf_pc.tile_lo : 0;
                            prefetch_next(false);  // this tile: loaded now
                            for (int i = 1; i < args.prefetch_tiles; ++i) prefetch_next(true);
                        }
                        prefetch_next(true);
                        // the tile's 9 chunks of E4M3 codes (rope first, as the MMAs use them)
                        for (int cc = 0; cc < kNumChunks; ++cc) {
                            const int c = (cc == 0) ? kNumChunks - 1 : cc - 1;
                            const uint32_t s = f8_cnt % C::NF;
                            ok = ptx::mbar_wait_bounded(f8_empty + s, ((f8_cnt / C::NF) & 1) ^ 1, tmo);
                            if (!ok) break;
                            ptx::mbar_arrive_expect_tx(f8_full + s, C::kF8Bytes);
                            if (!(blockIdx.x == 0 && unit == args.stall_unit))
                                ptx::tma_load_3d(f8_smem + s * C::kF8Bytes, &tm_kv, f8_full + s, c * kChunk, row0,
                                                 pc.b);
                            ++unit;
                            ++f8_cnt;
                        }
                        continue;
                    }
                    {
                        const uint32_t s = rope_cnt % C::NR;
                        ok = ptx::mbar_wait_bounded(rope_empty + s, ((rope_cnt / C::NR) & 1) ^ 1, tmo);
                        if (!ok) break;
                        ptx::mbar_arrive_expect_tx(rope_full + s, C::kChunkBytes);
                        if (!(blockIdx.x == 0 && unit == args.stall_unit))
                            ptx::tma_load_3d(rope_smem + s * C::kChunkBytes, &tm_kv, rope_full + s, 8 * kChunk,
                                             row0, pc.b);
                        ++unit;
                        ++rope_cnt;
                    }
                    for (int pp = 0; pp < 4; ++pp) {
                        const uint32_t s = pair_cnt % C::NP;
                        ok = ptx::mbar_wait_bounded(pair_empty + s, ((pair_cnt / C::NP) & 1) ^ 1, tmo);
                        if (!ok) break;
                        ptx::mbar_arrive_expect_tx(pair_full + s, C::kPairBytes);
                        if (!(blockIdx.x == 0 && unit == args.stall_unit)) {
                            uint8_t* dst = pair_smem + s * C::kPairBytes;
                            ptx::tma_load_3d(dst, &tm_kv, pair_full + s, (2 * pp) * kChunk, row0, pc.b);
                            ptx::tma_load_3d(dst + C::kChunkBytes, &tm_kv, pair_full + s, (2 * pp + 1) * kChunk,
                                             row0, pc.b);
                        }
                        ++unit;
                        ++pair_cnt;
                    }
                }
                ++piece_cnt;
            }
            if (!ok) {
                atomicOr(args.status, kStatusTimeout);
                *abort_flag = 1;
            }
            // Drain: every load this thread armed must have landed before the
            // CTA can exit (bounded; a load that was never issued -- the test
            // stall -- just runs the bound out).
            if (piece_cnt > 0 || pair_cnt > 0 || f8_cnt > 0) {
                if (piece_cnt > 0) ptx::mbar_wait_bounded(q_full, (piece_cnt - 1) & 1, tmo);
                if constexpr (SH::kFp8) {
                    for (uint32_t i = 0; i < C::NF && i < f8_cnt; ++i) {
                        const uint32_t use = f8_cnt - 1 - i;
                        ptx::mbar_wait_bounded(f8_full + (use % C::NF), (use / C::NF) & 1, tmo);
                    }
                }
                for (uint32_t i = 0; i < C::NP && i < pair_cnt; ++i) {
                    const uint32_t use = pair_cnt - 1 - i;  // the last use of slot use % NP
                    ptx::mbar_wait_bounded(pair_full + (use % C::NP), (use / C::NP) & 1, tmo);
                }
                for (uint32_t i = 0; i < C::NR && i < rope_cnt; ++i) {
                    const uint32_t use = rope_cnt - 1 - i;
                    ptx::mbar_wait_bounded(rope_full + (use % C::NR), (use / C::NR) & 1, tmo);
                }
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ============================================================ MMA issuer
        if (ptx::elect_one()) {
            uint32_t pair_cnt = 0, rope_cnt = 0, piece_cnt = 0, tile_cnt = 0;
            bool ok = true;
            const uint32_t q_base = ptx::smem_u32(q_smem);
            const uint32_t pt_base = ptx::smem_u32(pt_smem);
            const uint32_t tm_S = tmem_base + C::kColS;
            Piece pc;
            while (ok && walker.next(pc)) {
                for (int t = pc.tile_lo; t < pc.tile_hi; ++t) {
                    const bool first = (t == pc.tile_lo);
                    const bool last = (t == pc.tile_hi - 1);
                    if (first) {
                        // FP8: Q after the converters narrowed it to f16
                        ok = ptx::mbar_wait_bounded(SH::kFp8 ? q_ready : q_full, piece_cnt & 1, tmo);
                        if (!ok) break;
                    }
                    if (SH::kMha) {
                        // ---------------- S^T = K . Q^T over the K pair, O^T += V^T . P^T over the V pair
                        const uint32_t ks = pair_cnt % C::NP, vs = (pair_cnt + 1) % C::NP;
                        ok = ptx::mbar_wait_bounded(pair_full + ks, (pair_cnt / C::NP) & 1, tmo);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        {
                            const uint32_t kbase = ptx::smem_u32(pair_smem + ks * C::kPairBytes);
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk) {
                                    const uint64_t da = ptx::make_smem_desc(kbase + h * C::kChunkBytes + kk * 32, 16,
                                                                            1024, ptx::Swizzle::B128);
                                    const uint64_t db = ptx::make_smem_desc(q_base + h * C::kQChunkBytes + kk * 32, 16,
                                                                            1024, ptx::Swizzle::B128);
                                    ptx::mma_bf16_ss(tm_S, da, db, C::kIdescS, (h | kk) ? 1u : 0u);
                                }
                            }
                        }
                        ptx::mma_commit(pair_empty + ks);
                        if (last) ptx::mma_commit(q_empty);
                        ptx::mma_commit(s_full);
                        ok = ptx::mbar_wait_bounded(p_full, tile_cnt & 1, tmo) &&
                             ptx::mbar_wait_bounded(pair_full + vs, ((pair_cnt + 1) / C::NP) & 1, tmo);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        {
                            const uint32_t vbase = ptx::smem_u32(pair_smem + vs * C::kPairBytes);
#pragma unroll
                            for (int kk = 0; kk < kTileKV / 16; ++kk) {
                                const uint64_t da =
                                    ptx::make_smem_desc(vbase + kk * 2048, C::kChunkBytes, 1024, ptx::Swizzle::B128);
                                const uint64_t db = ptx::make_smem_desc(pt_base + kk * 2 * C::kPTAtom, C::kPTBytes,
                                                                        C::kPTAtom, C::kPTSwz);
                                ptx::mma_bf16_ss(tmem_base, da, db, C::kIdescPV, (!first || kk > 0) ? 1u : 0u);
                            }
                        }
                        ptx::mma_commit(pair_empty + vs);
                        pair_cnt += 2;
                        if (last) ptx::mma_commit(pv_done);
                        ++tile_cnt;
                        continue;
                    }
                    // ---------------- S^T = K . Q^T  (rope chunk first, then the 8 value chunks)
                    const uint32_t rs = rope_cnt % C::NR;
                    ok = ptx::mbar_wait_bounded(rope_full + rs, (rope_cnt / C::NR) & 1, tmo);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    {
                        const uint32_t a0 = ptx::smem_u32(rope_smem + rs * C::kChunkBytes);
                        const uint32_t b0 = q_base + 8 * C::kQChunkBytes;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t da = ptx::make_smem_desc(a0 + kk * 32, 16, 1024, ptx::Swizzle::B128);
                            const uint64_t db = ptx::make_smem_desc(b0 + kk * 32, 16, 1024, ptx::Swizzle::B128);
                            ptx::mma_bf16_ss(tm_S, da, db, C::kIdescS, kk > 0 ? 1u : 0u);
                        }
                    }
                    ptx::mma_commit(rope_empty + rs);
                    ++rope_cnt;
                    uint32_t slots[4];
                    for (int pp = 0; pp < 4; ++pp) {
                        const uint32_t s = (pair_cnt + pp) % C::NP;
                        slots[pp] = s;
                        ok = ptx::mbar_wait_bounded(pair_full + s, ((pair_cnt + pp) / C::NP) & 1, tmo);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        const uint32_t pbase = ptx::smem_u32(pair_smem + s * C::kPairBytes);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int c = 2 * pp + h;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint64_t da = ptx::make_smem_desc(pbase + h * C::kChunkBytes + kk * 32, 16,
                                                                        1024, ptx::Swizzle::B128);
                                const uint64_t db = ptx::make_smem_desc(q_base + c * C::kQChunkBytes + kk * 32, 16,
                                                                        1024, ptx::Swizzle::B128);
                                ptx::mma_bf16_ss(tm_S, da, db, C::kIdescS, 1u);
                            }
                        }
                    }
                    if (!ok) break;
                    if (last) ptx::mma_commit(q_empty);
                    ptx::mma_commit(s_full);
                    // ---------------- O^T += V^T . P^T  (after the softmax wrote P^T)
                    ok = ptx::mbar_wait_bounded(p_full, tile_cnt & 1, tmo);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    for (int pp = 0; pp < 4; ++pp) {
                        const uint32_t vbase = ptx::smem_u32(pair_smem + slots[pp] * C::kPairBytes);
                        const uint32_t tm_O = tmem_base + pp * G;
#pragma unroll
                        for (int kk = 0; kk < kTileKV / 16; ++kk) {
                            // A = V^T block: M = 128 dv (two 64-wide atoms 16 KB apart), K = 16 kv rows
                            const uint64_t da =
                                ptx::make_smem_desc(vbase + kk * 2048, C::kChunkBytes, 1024, ptx::Swizzle::B128);
                            // B = P^T: K = 16 kv rows (two 8-row atoms), N = G (one atom wide)
                            const uint64_t db = ptx::make_smem_desc(pt_base + kk * 2 * C::kPTAtom, C::kPTBytes,
                                                                    C::kPTAtom, C::kPTSwz);
                            ptx::mma_bf16_ss(tm_O, da, db, C::kIdescPV, (!first || kk > 0) ? 1u : 0u);
                        }
                        ptx::mma_commit(pair_empty + slots[pp]);
                    }
                    pair_cnt += 4;
                    if (last) ptx::mma_commit(pv_done);
                    ++tile_cnt;
                }
                ++piece_cnt;
            }
            if (!ok) {
                atomicOr(args.status, kStatusTimeout);
                *abort_flag = 1;
            }
            // drain: all MMAs this thread issued must complete before TMEM is freed
            ptx::mma_commit(drain);
            ptx::mbar_wait_bounded(drain, 0, tmo);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ============================================================ softmax + epilogue (warps 0-3)
        const int row_in_tile = warp * 32 + lane;            // TMEM lane = kv row (S^T) = dv row (O^T)
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
        const int my_col = col_of_lane<G>(lane);
        const bool writes_col = (G == 32) || ((lane & 1) == 0);
        uint32_t tile_cnt = 0, piece_cnt = 0, sync_cnt = 0;
        bool ok = true;
        // bounded barrier over the 128 softmax threads
        auto group_barrier = [&]() -> bool {
            ptx::mbar_arrive(group_sync);
            const bool r = ptx::mbar_wait_bounded(group_sync, sync_cnt & 1, tmo);
            ++sync_cnt;
            return r;
        };
        Piece pc;
        while (ok && walker.next(pc)) {
            float m_ref[G];
            float l_part[G];
#pragma unroll
            for (int j = 0; j < G; ++j) {
                m_ref[j] = -INFINITY;
                l_part[j] = 0.f;
            }
            for (int t = pc.tile_lo; t < pc.tile_hi; ++t) {
                const bool first = (t == pc.tile_lo);
                int row0 = t * kTileKV;
                if (row0 + kTileKV > pc.L) row0 = pc.L - kTileKV;
                const int kv_row = row0 + row_in_tile;
                const bool valid = (kv_row >= t * kTileKV) && (kv_row < pc.L);

                ok = ptx::mbar_wait_bounded(s_full, tile_cnt & 1, tmo);
                if (!ok) break;
                ptx::tc_fence_after();
                float x[G];
                {
                    uint32_t r[16];
#pragma unroll
                    for (int c0 = 0; c0 < G; c0 += 16) {
                        ptx::tmem_ld_16(lane_addr + C::kColS + c0, r);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            x[c0 + j] = valid ? __uint_as_float(r[j]) * args.scale_log2 : -INFINITY;
                    }
                }
                // column max over the tile's 128 kv rows
                float* redmax = red + (tile_cnt & 1) * 4 * G;
                const float wmax = warp_reduce_scatter<G, true>(x, lane);
                if (writes_col) redmax[warp * G + my_col] = wmax;
                ok = group_barrier();
                if (!ok) break;
                float tmax[G];
#pragma unroll
                for (int j = 0; j < G; j += 4) {
                    float4 a = *reinterpret_cast<const float4*>(redmax + 0 * G + j);
                    const float4 b1 = *reinterpret_cast<const float4*>(redmax + 1 * G + j);
                    const float4 b2 = *reinterpret_cast<const float4*>(redmax + 2 * G + j);
                    const float4 b3 = *reinterpret_cast<const float4*>(redmax + 3 * G + j);
                    tmax[j + 0] = fmaxf(fmaxf(a.x, b1.x), fmaxf(b2.x, b3.x));
                    tmax[j + 1] = fmaxf(fmaxf(a.y, b1.y), fmaxf(b2.y, b3.y));
                    tmax[j + 2] = fmaxf(fmaxf(a.z, b1.z), fmaxf(b2.z, b3.z));
                    tmax[j + 3] = fmaxf(fmaxf(a.w, b1.w), fmaxf(b2.w, b3.w));
                }
                // Lazy rescale: keep the reference max unless some column grew
                // by more than 8 (p <= 2^8 then); the decision is identical in
                // every thread (same shared data), so the branch is uniform.
                bool grow = false;
#pragma unroll
                for (int j = 0; j < G; ++j) grow |= (tmax[j] > m_ref[j] + 8.f);
                if (first) {
#pragma unroll
                    for (int j = 0; j < G; ++j) m_ref[j] = tmax[j];
                } else if (grow) {
                    float alpha[G];
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        const float mn = fmaxf(m_ref[j], tmax[j]);
                        alpha[j] = ex2_approx(m_ref[j] - mn);
                        m_ref[j] = mn;
                        l_part[j] *= alpha[j];
                    }
                    // O^T columns j *= alpha[j]; PV of the previous tile has
                    // completed (it was committed before this tile's S^T).
#pragma unroll
                    for (int blk = 0; blk < SH::kDvBlocks; ++blk) {
#pragma unroll
                        for (int c0 = 0; c0 < G; c0 += 16) {
                            uint32_t r[16];
                            ptx::tmem_ld_16(lane_addr + blk * G + c0, r);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 16; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha[c0 + j]);
                            ptx::tmem_st_16(lane_addr + blk * G + c0, r);
                        }
                    }
                    ptx::tmem_wait_st();
                }
                // P^T row for this kv row: G bf16 values, swizzled MN-major
                uint32_t packed[G / 2];
#pragma unroll
                for (int j = 0; j < G; j += 2) {
                    const float p0 = ex2_approx(x[j] - m_ref[j]);
                    const float p1 = ex2_approx(x[j + 1] - m_ref[j + 1]);
                    l_part[j] += p0;
                    l_part[j + 1] += p1;
                    if constexpr (SH::kFp8) {
                        const __half2 h2 = __floats2half2_rn(p0, p1);
                        packed[j / 2] = *reinterpret_cast<const uint32_t*>(&h2);
                    } else {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                        packed[j / 2] = *reinterpret_cast<const uint32_t*>(&h2);
                    }
                }
#pragma unroll
                for (int u = 0; u < (2 * G) / 16; ++u) {
                    const uint32_t off = swz_offset(row_in_tile, u, 2 * G);
                    *reinterpret_cast<uint4*>(pt_smem + off) =
                        make_uint4(packed[4 * u + 0], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                ptx::mbar_arrive(p_full);
                ++tile_cnt;
            }
            if (!ok) break;
            // ---------------- epilogue: O / l -> out (or a partial), lse
            ok = ptx::mbar_wait_bounded(pv_done, piece_cnt & 1, tmo);
            if (!ok) break;
            ptx::tc_fence_after();
            float* redsum = red + 8 * G;
            {
                const float ws = warp_reduce_scatter<G, false>(l_part, lane);
                if (writes_col) redsum[warp * G + my_col] = ws;
            }
            ok = group_barrier();
            if (!ok) break;
            // MHA: columns past Sq * gq are padding
            const int n_cols = SH::kMha ? args.Sq * (args.H / args.Hkv) : G;
            // a sink applies once per row: to whole sequences here, to cut ones in the combine
            const bool sink_here = (args.sinks != nullptr) && (pc.slot < 0);
            // thread j < G finishes query row j (sum, sink, lse) and leaves its
            // 1 / l in the max buffer the piece's last tile did not use
            float* fin = red + (tile_cnt & 1) * 4 * G;
            if (row_in_tile < n_cols) {
                const int j = row_in_tile;
                const int qr = group_row<SH>(args, G, g, j);  // query row within the sequence
                float mj = 0.f;
#pragma unroll
                for (int jj = 0; jj < G; ++jj)
                    if (jj == j) mj = m_ref[jj];
                float lj = redsum[0 * G + j] + redsum[1 * G + j] + redsum[2 * G + j] + redsum[3 * G + j];
                float c = 1.f;
                if (sink_here) c = fold_sink(mj, lj, args.sinks[qr % args.H] * kLog2e);
                fin[j] = c / lj * args.o_scale;
                const float lse_nat = (mj + log2f(lj)) * 0.69314718055994530942f;
                if (pc.slot < 0)
                    args.lse[static_cast<size_t>(pc.b) * args.R + qr] = lse_nat;
                else
                    args.part_lse[static_cast<size_t>(pc.slot) * args.R + qr] = lse_nat;
            }
            ok = group_barrier();
            if (!ok) break;
#pragma unroll
            for (int blk = 0; blk < SH::kDvBlocks; ++blk) {
                const int dv = blk * 128 + row_in_tile;
#pragma unroll
                for (int c0 = 0; c0 < G; c0 += 16) {
                    uint32_t r[16];
                    ptx::tmem_ld_16(lane_addr + blk * G + c0, r);
                    ptx::tmem_wait_ld();
                    if (pc.slot < 0) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            if (c0 + j >= n_cols) continue;
                            const size_t orow = static_cast<size_t>(pc.b) * args.R + group_row<SH>(args, G, g, c0 + j);
                            args.out[orow * SH::kDv + dv] = __float2bfloat16_rn(__uint_as_float(r[j]) * fin[c0 + j]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            if (c0 + j >= n_cols) continue;
                            const size_t orow =
                                static_cast<size_t>(pc.slot) * args.R + group_row<SH>(args, G, g, c0 + j);
                            args.part_o[orow * SH::kDv + dv] = __uint_as_float(r[j]) * fin[c0 + j];
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            // the next piece reuses the sums buffer only after everyone read it
            ok = group_barrier();
            ++piece_cnt;
        }
        if (!ok) {
            atomicOr(args.status, kStatusTimeout);
            *abort_flag = 1;
        }
    } else if (warp >= 6) {
        // ============================================================ FP8 converters (warps 6..)
        if constexpr (SH::kFp8) {
            const uint32_t r = threadIdx.x - 192;  // first kv row of the tile this thread widens
            uint32_t f8_cnt = 0, pair_cnt = 0, rope_cnt = 0, piece_cnt = 0;
            bool ok = true;
            Piece pc;
            while (ok && walker.next(pc)) {
                // this piece's Q rows: bf16 -> f16 in place (same element positions)
                ok = ptx::mbar_wait_bounded(q_full, piece_cnt & 1, tmo);
                if (!ok) break;
                for (uint32_t i = r; i < kNumChunks * C::kQChunkBytes / 16; i += C::kConvThreads) {
                    uint4* qp = reinterpret_cast<uint4*>(q_smem) + i;
                    *qp = bf16x8_to_f16x8(*qp);
                }
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(q_ready);
                for (int t = pc.tile_lo; t < pc.tile_hi && ok; ++t) {
                    for (int cc = 0; cc < kNumChunks; ++cc) {
                        const int c = (cc == 0) ? kNumChunks - 1 : cc - 1;
                        const uint32_t fs = f8_cnt % C::NF;
                        ok = ptx::mbar_wait_bounded(f8_full + fs, (f8_cnt / C::NF) & 1, tmo);
                        if (!ok) break;
                        uint8_t* dst;
                        if (c == kNumChunks - 1) {
                            const uint32_t rs = rope_cnt % C::NR;
                            ok = ptx::mbar_wait_bounded(rope_empty + rs, ((rope_cnt / C::NR) & 1) ^ 1, tmo);
                            dst = rope_smem + rs * C::kChunkBytes;
                        } else {
                            const uint32_t ps = pair_cnt % C::NP;
                            if ((c & 1) == 0)
                                ok = ptx::mbar_wait_bounded(pair_empty + ps, ((pair_cnt / C::NP) & 1) ^ 1, tmo);
                            dst = pair_smem + ps * C::kPairBytes + (c & 1) * C::kChunkBytes;
                        }
                        if (!ok) break;
#pragma unroll
                        for (uint32_t row = r; row < kTileKV; row += C::kConvThreads)
                            widen_chunk_row(f8_smem + fs * C::kF8Bytes, dst, row);
                        ptx::mbar_arrive(f8_empty + fs);  // codes read: the slot may be reloaded
                        // an operand slot is complete: publish it to the tensor core
                        if (c == kNumChunks - 1) {
                            ptx::fence_proxy_async_smem();
                            ptx::mbar_arrive(rope_full + rope_cnt % C::NR);
                            ++rope_cnt;
                        } else if (c & 1) {
                            ptx::fence_proxy_async_smem();
                            ptx::mbar_arrive(pair_full + pair_cnt % C::NP);
                            ++pair_cnt;
                        }
                        ++f8_cnt;
                    }
                }
                ++piece_cnt;
            }
            if (!ok) {
                atomicOr(args.status, kStatusTimeout);
                *abort_flag = 1;
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc<C::kTmemCols>(tmem_base);
    }
}

}  // namespace mla
