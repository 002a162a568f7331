// mla_decode.cu -- host side of the C ABI declared in include/mla_decode.h:
// argument validation, plan selection, TMA descriptor encoding and kernel
// launches.  The device code lives in the kernel_*.cuh headers.
//
// The driver entry point for TMA descriptors (cuTensorMapEncodeTiled) is
// fetched through the runtime (cudaGetDriverEntryPoint), so the library links
// the CUDA runtime statically and does not link libcuda directly: it loads on
// machines without a GPU driver (symbol checks), and fails with MLA_ERR_CUDA
// only when a call actually needs the device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/mla_decode.h"
#include "kernel_combine.cuh"
#include "kernel_pair_fp8.cuh"
#include "kernel_pair.cuh"
#include "kernel_transposed.cuh"
#include "kernel_fp8mma.cuh"

namespace {

constexpr size_t kHeaderBytes = 256;     // workspace status words
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s

std::atomic<unsigned long long> g_timeout_ns{0};
std::atomic<int> g_stall_unit{-1};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

struct Layout {
    size_t part_lse_off, part_o_off, total;
};

// partial slots: 2 per partition (balanced schedule), or one per S-tile chunk
// of every sequence at its longest (batch-invariant schedule)
long long num_slots(const mla_plan& pl) {
    if (pl.split_tiles > 0) {
        const long long tiles = (static_cast<long long>(pl.L_max) + mla::kTileKV - 1) / mla::kTileKV;
        return static_cast<long long>(pl.B) * ((tiles + pl.split_tiles - 1) / pl.split_tiles);
    }
    return 2LL * pl.num_partitions;
}

Layout workspace_layout(long long slots, int R, int dv = mla::kDv) {
    Layout l;
    l.part_lse_off = kHeaderBytes;
    l.part_o_off = align_up(l.part_lse_off + size_t(slots) * R * sizeof(float), 256);
    l.total = l.part_o_off + size_t(slots) * R * dv * sizeof(float);
    return l;
}

template <int G, class SH = mla::MlaShape>
mla_status launch_transposed(const mla_plan& plan, const CUtensorMap& tm_q, const CUtensorMap& tm_kv,
                             const CUtensorMap& tm_v, const mla::MainArgs& args, cudaStream_t stream) {
    using C = mla::TransposedCfg<G, SH>;
    auto kern = mla::mla_decode_transposed_kernel<G, SH>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
        return MLA_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(plan.num_partitions * plan.num_groups));
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(tm_q, tm_kv, tm_v, args);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

template <int G>
mla_status launch_fp8mma(const mla_plan& plan, const CUtensorMap& tm_kv, const mla::MainArgs& args,
                         cudaStream_t stream) {
    using C = mla::Fp8MmaCfg<G>;
    auto kern = mla::mla_decode_fp8mma_kernel<G>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
        return MLA_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(plan.num_partitions * plan.num_groups));
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(tm_kv, args);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int choose_group_rows(int R) {
    if (R == 16) return 16;
    return (R % 32 == 0) ? 32 : 16;
}

// pair-kernel ring depths: K chunks (8 KB each), V slots (32 KB each) and S
// buffers in TMEM (PV trails S by kPairNS - 1 tiles)
#ifndef MLA_PAIR_NK
#define MLA_PAIR_NK 7
#endif
#ifndef MLA_PAIR_NV
#define MLA_PAIR_NV 2
#endif
#ifndef MLA_PAIR_NS
#define MLA_PAIR_NS 3
#endif
#ifndef MLA_PAIR_NP
#define MLA_PAIR_NP 2
#endif
constexpr int kPairNK = MLA_PAIR_NK;
constexpr int kPairNV = MLA_PAIR_NV;
constexpr int kPairNS = MLA_PAIR_NS;
constexpr int kPairNP = MLA_PAIR_NP;  // P buffers in shared memory
constexpr int kDefaultPrefetchTiles = 1;

constexpr int kDefaultSplitTiles = 16;  // batch-invariant chunks: 16 tiles = 2048 keys
using PairC = mla::PairCfg<kPairNK, kPairNV, kPairNS, kPairNP>;

mla_status launch_pair(const mla_plan& plan, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                       const CUtensorMap& tm_v, const CUtensorMap& tm_pf, const CUtensorMap& tm_out,
                       const CUtensorMap& tm_part, const mla::MainArgs& args, cudaStream_t stream) {
    auto kern = mla::mla_decode_pair_kernel<kPairNK, kPairNV, kPairNS, kPairNP>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PairC::kSmemBytes) != cudaSuccess)
        return MLA_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(2 * plan.num_partitions * plan.num_groups));
    kern<<<grid, PairC::kThreads, PairC::kSmemBytes, stream>>>(tm_q, tm_k, tm_v, tm_pf, tm_out, tm_part, args);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

constexpr int kPairFp8NK = 18;  // K chunks of 4 KB (two tiles)
constexpr int kPairFp8NV = 3;   // V slots of 16 KB (a tile and a half)
using PairFp8C = mla::PairFp8Cfg<kPairFp8NK, kPairFp8NV, kPairNS, kPairNP>;

mla_status launch_pair_fp8(const mla_plan& plan, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                           const CUtensorMap& tm_pf, const CUtensorMap& tm_out, const CUtensorMap& tm_part,
                           const mla::MainArgs& args, cudaStream_t stream) {
    auto kern = mla::mla_decode_pair_fp8_kernel<kPairFp8NK, kPairFp8NV, kPairNS, kPairNP>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PairFp8C::kSmemBytes) != cudaSuccess)
        return MLA_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(2 * plan.num_partitions * plan.num_groups));
    kern<<<grid, PairFp8C::kThreads, PairFp8C::kSmemBytes, stream>>>(tm_k, tm_v, tm_pf, tm_out, tm_part, args);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// Output maps of the pair kernel's TMA-store epilogue: rows of 512 values,
// boxes of 32 rows x 128 bytes (64 bf16 or 32 fp32 columns), 128-byte swizzle.
bool encode_rows_store(EncodeTiledFn enc, CUtensorMap* m, const void* base, uint64_t rows, bool fp32) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(mla::kDv), rows};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(mla::kDv) * (fp32 ? 4 : 2)};
    const cuuint32_t box[2] = {fp32 ? 32u : 64u, 32u};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The combine kernel is a programmatic dependent of the main kernel before it
// on the stream: its CTAs may start (and scan the lengths) while the main
// kernel finishes, and wait in the kernel for the main grid's results.
template <int DV>
mla_status launch_combine(dim3 grid, const mla::CombineArgs& c, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(mla::kCombineThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mla::mla_decode_combine_kernel<DV>, c) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

bool encode_2d_bf16(EncodeTiledFn enc, CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                    uint32_t box_inner, uint32_t box_rows) {
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// kv viewed as [B][L_max][576]: a box of box_rows rows x 64 columns of one sequence
bool encode_kv(EncodeTiledFn enc, CUtensorMap* m, const void* kv, int L_max, int B, uint32_t box_rows) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(mla::kDqk), static_cast<cuuint64_t>(L_max),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(mla::kDqk) * 2,
                                   static_cast<cuuint64_t>(mla::kDqk) * 2 * L_max};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(mla::kChunk), box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// kv viewed with its 64-column chunks as an outer dimension: [B][9 chunks][L_max][64],
// strides 1152 * L_max, 128, 1152 bytes.  A box of box_rows rows x box_chunks
// adjacent chunks lands in shared memory chunk after chunk, each chunk a
// [box_rows][64] block in the same 128-byte swizzle a single-chunk box gives.
bool encode_kv_chunks(EncodeTiledFn enc, CUtensorMap* m, const void* kv, int L_max, int B, uint32_t box_rows,
                      uint32_t box_chunks) {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(mla::kChunk), static_cast<cuuint64_t>(L_max),
                                static_cast<cuuint64_t>(mla::kNumChunks), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(mla::kDqk) * 2, static_cast<cuuint64_t>(mla::kChunk) * 2,
                                   static_cast<cuuint64_t>(mla::kDqk) * 2 * L_max};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(mla::kChunk), box_rows, box_chunks, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(kv), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q viewed as [9 chunks][rows][64] (strides 128, 1152 bytes): one box holds
// 64 rows x all 9 chunks, chunk after chunk
bool encode_q_chunks(EncodeTiledFn enc, CUtensorMap* m, const void* q, uint64_t rows) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(mla::kChunk), rows, static_cast<cuuint64_t>(mla::kNumChunks)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(mla::kDqk) * 2, static_cast<cuuint64_t>(mla::kChunk) * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(mla::kChunk), 64, static_cast<cuuint32_t>(mla::kNumChunks)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP8 cache: kv viewed as [B][L_max][576] bytes (E4M3 codes): a box of
// box_rows rows x 64 codes, 64-byte swizzle (rows of 64 bytes).  The FP8 maps
// promote L2 fills in 128-byte steps: with 256 bytes per 64-byte row segment
// the low-head decode ran 6 % slower (L2 was its busiest unit).
bool encode_kv_fp8(EncodeTiledFn enc, CUtensorMap* m, const void* kv, int L_max, int B, uint32_t box_rows) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(mla::kDqk), static_cast<cuuint64_t>(L_max),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(mla::kDqk),
                                   static_cast<cuuint64_t>(mla::kDqk) * L_max};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(mla::kChunk), box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(kv), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP8 cache with its 64-code chunks as an outer dimension: [B][9 chunks][L_max][64]
// bytes, strides 576 * L_max, 64, 576.  A box of box_rows rows x box_chunks
// adjacent chunks lands chunk after chunk, each a [box_rows][64] block in the
// 64-byte swizzle a single-chunk box gives.
bool encode_kv_fp8_chunks(EncodeTiledFn enc, CUtensorMap* m, const void* kv, int L_max, int B, uint32_t box_rows,
                          uint32_t box_chunks) {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(mla::kChunk), static_cast<cuuint64_t>(L_max),
                                static_cast<cuuint64_t>(mla::kNumChunks), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(mla::kDqk), static_cast<cuuint64_t>(mla::kChunk),
                                   static_cast<cuuint64_t>(mla::kDqk) * L_max};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(mla::kChunk), box_rows, box_chunks, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(kv), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

int32_t mla_decode_abi_version(void) { return 10000; }

const char* mla_status_string(mla_status s) {
    switch (s) {
        case MLA_OK: return "ok";
        case MLA_ERR_INVALID_ARG: return "invalid argument";
        case MLA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case MLA_ERR_UNSUPPORTED: return "unsupported shape or device (needs sm_100)";
        case MLA_ERR_CUDA: return "CUDA call failed";
        case MLA_ERR_TIMEOUT: return "device pipeline wait timed out; results invalid";
        case MLA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case MLA_ERR_SEQLEN: return "a sequence length was outside [0, L_max] (clamped)";
    }
    return "unknown status";
}

mla_status mla_decode_plan(int32_t B, int32_t Sq, int32_t H, int32_t L_max, int32_t device,
                           int32_t num_partitions_override, mla_plan* plan, size_t* workspace_bytes) {
    return mla_decode_plan_kernel(B, Sq, H, L_max, device, num_partitions_override, 0, plan, workspace_bytes);
}

mla_status mla_decode_plan_kernel(int32_t B, int32_t Sq, int32_t H, int32_t L_max, int32_t device,
                                  int32_t num_partitions_override, int32_t kernel, mla_plan* plan,
                                  size_t* workspace_bytes) {
    if (!plan) return MLA_ERR_INVALID_ARG;
    if (kernel != 0 && kernel != MLA_KERNEL_TRANSPOSED && kernel != MLA_KERNEL_PAIR) return MLA_ERR_INVALID_ARG;
    if (B < 1 || B > 65535 || Sq < 1 || Sq > 16 || L_max < 1 || L_max > (1 << 24)) return MLA_ERR_INVALID_ARG;
    if (H != 16 && H != 32 && H != 64 && H != 128) return MLA_ERR_UNSUPPORTED;
    if (num_partitions_override < 0) return MLA_ERR_INVALID_ARG;
    int sms = 148;  // device < 0: plan for a B200 without touching a device
    if (device >= 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
            cudaGetLastError();
            return MLA_ERR_CUDA;
        }
    }
    mla_plan p;
    std::memset(&p, 0, sizeof p);
    p.B = B;
    p.Sq = Sq;
    p.H = H;
    p.L_max = L_max;
    p.device = device;
    p.num_sms = sms;
    const int R = Sq * H;
    if (kernel == 0) kernel = (R % 128 == 0) ? MLA_KERNEL_PAIR : MLA_KERNEL_TRANSPOSED;
    if (kernel == MLA_KERNEL_PAIR && R % 128 != 0) return MLA_ERR_UNSUPPORTED;
    p.kernel = kernel;
    int ctas_per_partition;
    if (kernel == MLA_KERNEL_PAIR) {
        p.group_rows = 128;
        p.num_groups = R / 128;
        p.cta_threads = PairC::kThreads;
        p.smem_bytes = PairC::kSmemBytes;
        ctas_per_partition = 2 * p.num_groups;
    } else {
        const int G = choose_group_rows(R);
        p.group_rows = G;
        p.num_groups = R / G;
        p.cta_threads = 192;
        p.smem_bytes = (G == 16) ? mla::TransposedCfg<16>::kSmemBytes : mla::TransposedCfg<32>::kSmemBytes;
        ctas_per_partition = p.num_groups;
    }
    int P = num_partitions_override > 0 ? num_partitions_override : sms / ctas_per_partition;
    if (P < 1) P = 1;
    if (P > 4096) P = 4096;
    p.num_partitions = P;
    p.tile_kv = mla::kTileKV;
    p.l2_prefetch_tiles = kDefaultPrefetchTiles;
    p.split_tiles = 0;
    p.Hkv = 1;
    p.head_dim = mla::kDqk;
    p.workspace_bytes = workspace_layout(num_slots(p), R).total;
    *plan = p;
    if (workspace_bytes) *workspace_bytes = p.workspace_bytes;
    return MLA_OK;
}

mla_status mla_decode_plan_batch_invariant(int32_t B, int32_t Sq, int32_t H, int32_t L_max, int32_t device,
                                           int32_t split_tiles, mla_plan* plan, size_t* workspace_bytes) {
    if (!plan) return MLA_ERR_INVALID_ARG;
    if (split_tiles == 0) split_tiles = kDefaultSplitTiles;
    if (split_tiles < 1 || split_tiles > (1 << 17)) return MLA_ERR_INVALID_ARG;
    mla_plan p;
    const mla_status st = mla_decode_plan_kernel(B, Sq, H, L_max, device, 0, 0, &p, nullptr);
    if (st != MLA_OK) return st;
    p.split_tiles = split_tiles;
    p.workspace_bytes = workspace_layout(num_slots(p), Sq * H).total;
    *plan = p;
    if (workspace_bytes) *workspace_bytes = p.workspace_bytes;
    return MLA_OK;
}

mla_status mla_decode_plan_fp8(int32_t B, int32_t Sq, int32_t H, int32_t L_max, int32_t device,
                               int32_t num_partitions_override, mla_plan* plan, size_t* workspace_bytes) {
    return mla_decode_plan_fp8_kernel(B, Sq, H, L_max, device, num_partitions_override, 0, plan, workspace_bytes);
}

mla_status mla_decode_plan_fp8_kernel(int32_t B, int32_t Sq, int32_t H, int32_t L_max, int32_t device,
                                      int32_t num_partitions_override, int32_t kernel, mla_plan* plan,
                                      size_t* workspace_bytes) {
    if (!plan) return MLA_ERR_INVALID_ARG;
    // default: the codes as kind::f8f6f4 operands; on a CTA pair when Sq * H is a
    // multiple of 128 (1.4x the transposed operand kernel there), else the
    // transposed operand kernel (2.3x the widening kernel on a B200)
    if (kernel == 0) kernel = ((Sq * H) % 128 == 0) ? MLA_KERNEL_FP8_PAIR : MLA_KERNEL_FP8_MMA;
    if (kernel != MLA_KERNEL_FP8 && kernel != MLA_KERNEL_FP8_MMA && kernel != MLA_KERNEL_FP8_PAIR)
        return MLA_ERR_INVALID_ARG;
    mla_plan p;
    const mla_status st = mla_decode_plan_kernel(B, Sq, H, L_max, device, num_partitions_override,
                                                 kernel == MLA_KERNEL_FP8_PAIR ? MLA_KERNEL_PAIR : MLA_KERNEL_TRANSPOSED,
                                                 &p, nullptr);
    if (st != MLA_OK) return st;
    p.kernel = kernel;
    if (kernel == MLA_KERNEL_FP8_PAIR) {  // the pair plan's groups and partitions
        p.cta_threads = PairFp8C::kThreads;
        p.smem_bytes = PairFp8C::kSmemBytes;
        *plan = p;
        if (workspace_bytes) *workspace_bytes = p.workspace_bytes;
        return MLA_OK;
    }
    const bool g16 = (p.group_rows == 16);
    if (kernel == MLA_KERNEL_FP8) {
        p.cta_threads = g16 ? mla::TransposedCfg<16, mla::MlaFp8Shape>::kThreads
                            : mla::TransposedCfg<32, mla::MlaFp8Shape>::kThreads;
        p.smem_bytes = g16 ? mla::TransposedCfg<16, mla::MlaFp8Shape>::kSmemBytes
                           : mla::TransposedCfg<32, mla::MlaFp8Shape>::kSmemBytes;
    } else {
        p.cta_threads = mla::Fp8MmaCfg<16>::kThreads;
        p.smem_bytes = g16 ? mla::Fp8MmaCfg<16>::kSmemBytes : mla::Fp8MmaCfg<32>::kSmemBytes;
    }
    *plan = p;
    if (workspace_bytes) *workspace_bytes = p.workspace_bytes;
    return MLA_OK;
}

mla_status mla_decode_workspace_init(const mla_plan* plan, void* workspace, size_t workspace_bytes, void* stream) {
    if (!plan || !workspace) return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < plan->workspace_bytes || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
    if (cudaMemsetAsync(workspace, 0, kHeaderBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

}  // extern "C"

namespace {

// Host-side checks of a run's plan and arguments; touches no device and
// enqueues nothing.  kv_scale: null for a bf16 cache; for an FP8 cache (plan
// kind MLA_KERNEL_FP8) the host address of its dequantization scale.
mla_status check_run_args(const mla_plan* plan, const void* q, const void* kv, const int32_t* seqlens,
                          float softmax_scale, const float* sinks, const void* out, const float* lse, int phases,
                          const float* kv_scale) {
    if (phases < 1 || phases > 3) return MLA_ERR_INVALID_ARG;
    if (!plan || !q || !kv || !seqlens || !out || !lse) return MLA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
    const bool fp8 = (plan->kernel == MLA_KERNEL_FP8 || plan->kernel == MLA_KERNEL_FP8_MMA ||
                      plan->kernel == MLA_KERNEL_FP8_PAIR);
    if (fp8 != (kv_scale != nullptr)) return MLA_ERR_INVALID_ARG;  // plan kind and entry point disagree
    if (fp8 && !(std::isfinite(*kv_scale) && *kv_scale > 0.f)) return MLA_ERR_INVALID_ARG;
    const mla_plan& pl = *plan;
    const int R = pl.Sq * pl.H;
    if (pl.B < 1 || pl.Sq < 1 || pl.H < 1 || pl.L_max < 1 || pl.num_partitions < 1 || pl.num_groups < 1 ||
        pl.group_rows * pl.num_groups != R)
        return MLA_ERR_INVALID_ARG;
    if (pl.l2_prefetch_tiles < 0 || pl.l2_prefetch_tiles > 16) return MLA_ERR_INVALID_ARG;
    if (pl.split_tiles < 0 || pl.split_tiles > (1 << 17)) return MLA_ERR_INVALID_ARG;
    if (pl.kernel == MLA_KERNEL_TRANSPOSED || pl.kernel == MLA_KERNEL_FP8 || pl.kernel == MLA_KERNEL_FP8_MMA) {
        if (pl.group_rows != 16 && pl.group_rows != 32) return MLA_ERR_INVALID_ARG;
    } else if (pl.kernel == MLA_KERNEL_PAIR || pl.kernel == MLA_KERNEL_FP8_PAIR) {
        if (pl.group_rows != 128) return MLA_ERR_INVALID_ARG;
    } else {
        return MLA_ERR_INVALID_ARG;  // MHA plans run through mha_decode_run
    }
    if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(seqlens, 4) ||
        !aligned(sinks, 4))
        return MLA_ERR_ALIGNMENT;
    return MLA_OK;
}

// The current device must be the plan's (when the plan names one) and an sm_100 GPU.
mla_status check_run_device(const mla_plan& pl) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    if (pl.device >= 0 && dev != pl.device) return MLA_ERR_INVALID_ARG;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

// Encode the tensor maps and launch the requested phases; the arguments, the
// workspace and the device have been checked.
mla_status launch_phases(const mla_plan& pl, const void* q, const void* kv, const int32_t* seqlens,
                         float softmax_scale, const float* sinks, void* out, float* lse, void* workspace,
                         void* stream_, int phases, const float* kv_scale) {
    const bool fp8 = (pl.kernel == MLA_KERNEL_FP8 || pl.kernel == MLA_KERNEL_FP8_MMA || pl.kernel == MLA_KERNEL_FP8_PAIR);
    const int R = pl.Sq * pl.H;
    const Layout lay = workspace_layout(num_slots(pl), R);
    EncodeTiledFn enc = encode_fn();
    if (!enc) return MLA_ERR_CUDA;

    const int G = pl.group_rows;
    CUtensorMap tm_q, tm_kv, tm_k, tm_pf, tm_out, tm_part;
    if (pl.kernel == MLA_KERNEL_PAIR) {
        // Q: 64-row halves, all 9 chunks per box; K: one chunk of 64 own kv rows;
        // V: 2 chunks x all 128 rows of a tile; L2 prefetch: 64 rows x all 9
        // chunks; out and the fp32 partials: the epilogue's TMA stores
        uint8_t* part_o = static_cast<uint8_t*>(workspace) + lay.part_o_off;
        if (!encode_q_chunks(enc, &tm_q, q, static_cast<uint64_t>(pl.B) * R) ||
            !encode_kv(enc, &tm_k, kv, pl.L_max, pl.B, 64) ||
            !encode_kv_chunks(enc, &tm_kv, kv, pl.L_max, pl.B, mla::kTileKV, 2) ||
            !encode_kv_chunks(enc, &tm_pf, kv, pl.L_max, pl.B, 64, mla::kNumChunks) ||
            !encode_rows_store(enc, &tm_out, out, static_cast<uint64_t>(pl.B) * R, false) ||
            !encode_rows_store(enc, &tm_part, part_o, static_cast<uint64_t>(num_slots(pl)) * R, true))
            return MLA_ERR_CUDA;
    } else if (pl.kernel == MLA_KERNEL_FP8_PAIR) {
        // K: one 64-code chunk of 64 own kv rows; V: 2 chunks x all 128 rows of a
        // tile; L2 prefetch: 64 rows x all 9 chunks (64-byte swizzle); Q terms are
        // written by the kernel from q; out and the fp32 partials as for bf16
        uint8_t* part_o = static_cast<uint8_t*>(workspace) + lay.part_o_off;
        if (!encode_kv_fp8(enc, &tm_k, kv, pl.L_max, pl.B, 64) ||
            !encode_kv_fp8_chunks(enc, &tm_kv, kv, pl.L_max, pl.B, mla::kTileKV, 2) ||
            !encode_kv_fp8_chunks(enc, &tm_pf, kv, pl.L_max, pl.B, 64, mla::kNumChunks) ||
            !encode_rows_store(enc, &tm_out, out, static_cast<uint64_t>(pl.B) * R, false) ||
            !encode_rows_store(enc, &tm_part, part_o, static_cast<uint64_t>(num_slots(pl)) * R, true))
            return MLA_ERR_CUDA;
    } else if (fp8) {
        if (!encode_2d_bf16(enc, &tm_q, q, mla::kDqk, static_cast<uint64_t>(pl.B) * R, mla::kChunk, G) ||
            !encode_kv_fp8(enc, &tm_kv, kv, pl.L_max, pl.B, mla::kTileKV))
            return MLA_ERR_CUDA;
    } else {
        if (!encode_2d_bf16(enc, &tm_q, q, mla::kDqk, static_cast<uint64_t>(pl.B) * R, mla::kChunk, G) ||
            !encode_kv(enc, &tm_kv, kv, pl.L_max, pl.B, mla::kTileKV))
            return MLA_ERR_CUDA;
    }

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    mla::MainArgs a;
    a.seqlens = seqlens;
    a.B = pl.B;
    a.R = R;
    a.L_max = pl.L_max;
    a.P = pl.num_partitions;
    a.NG = pl.num_groups;
    // an FP8 cache's scale multiplies every key (scores) and every value (output
    // rows); the widening kernel's f16 operands hold the E4M3 values divided by
    // 2^8, the FP8-operand kernel multiplies the codes themselves
    const double kvs = !fp8 ? 1.0
                            : static_cast<double>(*kv_scale) *
                                  (pl.kernel == MLA_KERNEL_FP8 ? static_cast<double>(mla::kF8Unscale) : 1.0);
    a.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * kvs * 1.4426950408889634074);
    a.o_scale = static_cast<float>(kvs);
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.out = static_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.part_o = reinterpret_cast<float*>(ws + lay.part_o_off);
    a.part_lse = reinterpret_cast<float*>(ws + lay.part_lse_off);
    a.status = reinterpret_cast<uint32_t*>(ws);
    const unsigned long long tmo = g_timeout_ns.load();
    a.timeout_ns = tmo ? tmo : kDefaultTimeoutNs;
    a.stall_unit = g_stall_unit.load();
    a.prefetch_tiles = pl.l2_prefetch_tiles;
    a.sinks = sinks;
    a.H = pl.H;
    a.split_tiles = pl.split_tiles;
    a.Sq = pl.Sq;
    a.Hkv = 1;

    if (phases & 1) {
        mla_status st;
        if (pl.kernel == MLA_KERNEL_PAIR)
            st = launch_pair(pl, tm_q, tm_k, tm_kv, tm_pf, tm_out, tm_part, a, stream);
        else if (pl.kernel == MLA_KERNEL_FP8_PAIR)
            st = launch_pair_fp8(pl, tm_k, tm_kv, tm_pf, tm_out, tm_part, a, stream);
        else if (pl.kernel == MLA_KERNEL_FP8_MMA)
            st = (G == 16) ? launch_fp8mma<16>(pl, tm_kv, a, stream) : launch_fp8mma<32>(pl, tm_kv, a, stream);
        else if (fp8)
            st = (G == 16) ? launch_transposed<16, mla::MlaFp8Shape>(pl, tm_q, tm_kv, tm_kv, a, stream)
                           : launch_transposed<32, mla::MlaFp8Shape>(pl, tm_q, tm_kv, tm_kv, a, stream);
        else
            st = (G == 16) ? launch_transposed<16>(pl, tm_q, tm_kv, tm_kv, a, stream)
                           : launch_transposed<32>(pl, tm_q, tm_kv, tm_kv, a, stream);
        if (st != MLA_OK) {
            cudaGetLastError();
            return st;
        }
    }
    if (!(phases & 2)) return MLA_OK;
    mla::CombineArgs c;
    c.seqlens = seqlens;
    c.B = pl.B;
    c.R = R;
    c.L_max = pl.L_max;
    c.P = pl.num_partitions;
    c.out = a.out;
    c.lse = lse;
    c.part_o = a.part_o;
    c.part_lse = a.part_lse;
    c.sinks = sinks;
    c.H = pl.H;
    c.split_tiles = pl.split_tiles;
    const dim3 cgrid(static_cast<unsigned>(pl.B), static_cast<unsigned>(mla::combine_grid_y(pl.B, R, pl.num_sms)));
    return launch_combine<mla::kDv>(cgrid, c, stream);
}

mla_status run_phases(const mla_plan* plan, const void* q, const void* kv, const int32_t* seqlens,
                      float softmax_scale, const float* sinks, void* out, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream, int phases, const float* kv_scale = nullptr) {
    mla_status st = check_run_args(plan, q, kv, seqlens, softmax_scale, sinks, out, lse, phases, kv_scale);
    if (st != MLA_OK) return st;
    const Layout lay = workspace_layout(num_slots(*plan), plan->Sq * plan->H);
    if (!workspace || workspace_bytes < lay.total || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
    st = check_run_device(*plan);
    if (st != MLA_OK) return st;
    return launch_phases(*plan, q, kv, seqlens, softmax_scale, sinks, out, lse, workspace, stream, phases, kv_scale);
}

}  // namespace

extern "C" {

mla_status mla_decode_run(const mla_plan* plan, const void* q, const void* kv, const int32_t* seqlens,
                          float softmax_scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                          void* stream) {
    return run_phases(plan, q, kv, seqlens, softmax_scale, nullptr, out, lse, workspace, workspace_bytes, stream, 3);
}

mla_status mla_decode_run_sinks(const mla_plan* plan, const void* q, const void* kv, const int32_t* seqlens,
                                float softmax_scale, const float* sinks, void* out, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream) {
    return run_phases(plan, q, kv, seqlens, softmax_scale, sinks, out, lse, workspace, workspace_bytes, stream, 3);
}

mla_status mla_decode_run_phase(const mla_plan* plan, const void* q, const void* kv, const int32_t* seqlens,
                                float softmax_scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                                void* stream, int32_t phase) {
    if (phase != 1 && phase != 2) return MLA_ERR_INVALID_ARG;
    return run_phases(plan, q, kv, seqlens, softmax_scale, nullptr, out, lse, workspace, workspace_bytes, stream,
                      phase);
}

mla_status mla_decode_run_fp8(const mla_plan* plan, const void* q, const void* kv_fp8, float kv_scale,
                              const int32_t* seqlens, float softmax_scale, const float* sinks, void* out, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream) {
    return run_phases(plan, q, kv_fp8, seqlens, softmax_scale, sinks, out, lse, workspace, workspace_bytes, stream, 3,
                      &kv_scale);
}

mla_status mla_decode_run_fp8_phase(const mla_plan* plan, const void* q, const void* kv_fp8, float kv_scale,
                                    const int32_t* seqlens, float softmax_scale, void* out, float* lse,
                                    void* workspace, size_t workspace_bytes, void* stream, int32_t phase) {
    if (phase != 1 && phase != 2) return MLA_ERR_INVALID_ARG;
    return run_phases(plan, q, kv_fp8, seqlens, softmax_scale, nullptr, out, lse, workspace, workspace_bytes, stream,
                      phase, &kv_scale);
}

mla_status mla_decode_check(const mla_plan* plan, void* workspace, void* stream) {
    if (!plan || !workspace) return MLA_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    uint32_t st = 0;
    if (cudaMemcpy(&st, workspace, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(workspace, 0, sizeof st) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    if (st & mla::kStatusTimeout) return MLA_ERR_TIMEOUT;
    if (st & mla::kStatusSeqlen) return MLA_ERR_SEQLEN;
    return MLA_OK;
}

mla_status mla_decode_set_debug(uint64_t wait_timeout_ns, int32_t stall_tile) {
    g_timeout_ns.store(wait_timeout_ns);
    g_stall_unit.store(stall_tile < 0 ? -1 : stall_tile);
    return MLA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Run variant that allocates nothing: its split-KV partials and status words
// live in one file-scope device array instead of a caller workspace.  It is
// for callers that may not allocate device memory on the decode path, e.g. a
// serving engine that reserved nearly all HBM for its KV cache at start-up, or
// a C host with no device allocator of its own.  Every GPU that loads this
// library holds the array (MLA_NOALLOC_SCRATCH_BYTES) until the process exits.
// ---------------------------------------------------------------------------

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device `dev`.  The name
// g_noalloc_scratch is only a host-side handle; the address comes from
// cudaGetSymbolAddress, taken once per device while that device is current.
mla_status noalloc_scratch(int dev, void** ptr) {
    if (dev < 0 || dev >= kNoAllocMaxDevices) return MLA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MLA_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return MLA_OK;
}

}  // namespace

extern "C" {

mla_status mla_decode_run_noalloc(const mla_plan* plan, const void* q, const void* kv, const int32_t* seqlens,
                                  float softmax_scale, void* out, float* lse, int32_t wait_and_check,
                                  void* stream_) {
    // every check comes before anything is enqueued, so a rejected call leaves
    // the scratch (and an earlier call still running on it) untouched
    if (!plan) return MLA_ERR_INVALID_ARG;
    if (plan->num_partitions < 1 || plan->num_partitions > 4096 || plan->Sq < 1 || plan->H < 1)
        return MLA_ERR_INVALID_ARG;
    if (plan->split_tiles < 0 || plan->split_tiles > (1 << 17) || plan->B < 1 || plan->L_max < 1)
        return MLA_ERR_INVALID_ARG;
    mla_status st = check_run_args(plan, q, kv, seqlens, softmax_scale, nullptr, out, lse, 3, nullptr);
    if (st != MLA_OK) return st;
    const size_t need = workspace_layout(num_slots(*plan), plan->Sq * plan->H).total;
    if (need > MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
    st = check_run_device(*plan);
    if (st != MLA_OK) return st;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    void* scratch = nullptr;
    st = noalloc_scratch(dev, &scratch);
    if (st != MLA_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    // the status words must start at zero; the partial slots are always
    // written before they are read, so what an earlier call left there is
    // harmless
    if (cudaMemsetAsync(scratch, 0, kHeaderBytes, stream) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    st = launch_phases(*plan, q, kv, seqlens, softmax_scale, nullptr, out, lse, scratch, stream_, 3, nullptr);
    if (st != MLA_OK || !wait_and_check) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    uint32_t word = 0;
    if (cudaMemcpy(&word, scratch, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    if (word & mla::kStatusTimeout) return MLA_ERR_TIMEOUT;
    if (word & mla::kStatusSeqlen) return MLA_ERR_SEQLEN;
    return MLA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// MHA decode on the transposed kernel (MhaShape): q [B, Sq, H, 128], k and v
// [B, L_max, Hkv, 128]; one CTA per (partition, kv head).
// ---------------------------------------------------------------------------

namespace {

// a 4-D bf16 tensor, innermost dimension d[0] contiguous
bool encode_4d_bf16(EncodeTiledFn enc, CUtensorMap* m, const void* base, const uint64_t d[4], const uint32_t box[4]) {
    const cuuint64_t dims[4] = {d[0], d[1], d[2], d[3]};
    const cuuint64_t strides[3] = {d[0] * 2, d[0] * d[1] * 2, d[0] * d[1] * d[2] * 2};
    const cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, bx, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kMhaD = mla::MhaShape::kDv;  // 128: key and value width

}  // namespace

extern "C" {

mla_status mha_decode_plan(int32_t B, int32_t Sq, int32_t H, int32_t Hkv, int32_t L_max, int32_t device,
                           int32_t num_partitions_override, mla_plan* plan, size_t* workspace_bytes) {
    if (!plan) return MLA_ERR_INVALID_ARG;
    if (B < 1 || B > 65535 || Sq < 1 || Sq > 16 || L_max < 1 || L_max > (1 << 24) || H < 1 || Hkv < 1 ||
        H > 65535 || num_partitions_override < 0)
        return MLA_ERR_INVALID_ARG;
    if (H % Hkv != 0) return MLA_ERR_INVALID_ARG;
    const int gq = H / Hkv;
    if (Sq * gq > 32) return MLA_ERR_UNSUPPORTED;
    int sms = 148;
    if (device >= 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
            cudaGetLastError();
            return MLA_ERR_CUDA;
        }
    }
    mla_plan p;
    std::memset(&p, 0, sizeof p);
    p.B = B;
    p.Sq = Sq;
    p.H = H;
    p.L_max = L_max;
    p.device = device;
    p.num_sms = sms;
    p.kernel = MLA_KERNEL_MHA;
    p.group_rows = (Sq * gq <= 16) ? 16 : 32;
    p.num_groups = Hkv;
    p.cta_threads = 192;
    p.smem_bytes = (p.group_rows == 16) ? mla::TransposedCfg<16, mla::MhaShape>::kSmemBytes
                                        : mla::TransposedCfg<32, mla::MhaShape>::kSmemBytes;
    int P = num_partitions_override > 0 ? num_partitions_override : sms / Hkv;
    if (P < 1) P = 1;
    if (P > 4096) P = 4096;
    p.num_partitions = P;
    p.tile_kv = mla::kTileKV;
    p.l2_prefetch_tiles = 0;
    p.split_tiles = 0;
    p.Hkv = Hkv;
    p.head_dim = kMhaD;
    p.workspace_bytes = workspace_layout(num_slots(p), Sq * H, kMhaD).total;
    *plan = p;
    if (workspace_bytes) *workspace_bytes = p.workspace_bytes;
    return MLA_OK;
}

}  // extern "C"

namespace {

mla_status mha_run_phases(const mla_plan* plan, const void* q, const void* k, const void* v, const int32_t* seqlens,
                          float softmax_scale, const float* sinks, void* out, float* lse, void* workspace,
                          size_t workspace_bytes, void* stream_, int phases) {
    if (phases < 1 || phases > 3) return MLA_ERR_INVALID_ARG;
    if (!plan || !q || !k || !v || !seqlens || !out || !lse) return MLA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
    const mla_plan& pl = *plan;
    if (pl.kernel != MLA_KERNEL_MHA || pl.Hkv < 1 || pl.H < 1 || pl.H % pl.Hkv != 0 || pl.B < 1 || pl.Sq < 1 ||
        pl.L_max < 1 || pl.num_partitions < 1 || pl.num_groups != pl.Hkv || pl.head_dim != kMhaD ||
        pl.split_tiles < 0 || pl.split_tiles > (1 << 17))
        return MLA_ERR_INVALID_ARG;
    const int gq = pl.H / pl.Hkv;
    const int G = pl.group_rows;
    if ((G != 16 && G != 32) || pl.Sq * gq > G) return MLA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
        !aligned(seqlens, 4) || !aligned(sinks, 4))
        return MLA_ERR_ALIGNMENT;
    const int R = pl.Sq * pl.H;
    const Layout lay = workspace_layout(num_slots(pl), R, kMhaD);
    if (!workspace || workspace_bytes < lay.total || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    if (pl.device >= 0 && dev != pl.device) return MLA_ERR_INVALID_ARG;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return MLA_ERR_UNSUPPORTED;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return MLA_ERR_CUDA;

    CUtensorMap tm_q, tm_k, tm_v;
    {
        const uint64_t dq[4] = {static_cast<uint64_t>(kMhaD), static_cast<uint64_t>(pl.H),
                                static_cast<uint64_t>(pl.Sq), static_cast<uint64_t>(pl.B)};
        const uint32_t bq[4] = {static_cast<uint32_t>(mla::kChunk), static_cast<uint32_t>(gq),
                                static_cast<uint32_t>(pl.Sq), 1u};
        const uint64_t dk[4] = {static_cast<uint64_t>(kMhaD), static_cast<uint64_t>(pl.Hkv),
                                static_cast<uint64_t>(pl.L_max), static_cast<uint64_t>(pl.B)};
        const uint32_t bk[4] = {static_cast<uint32_t>(mla::kChunk), 1u, static_cast<uint32_t>(mla::kTileKV), 1u};
        if (!encode_4d_bf16(enc, &tm_q, q, dq, bq) || !encode_4d_bf16(enc, &tm_k, k, dk, bk) ||
            !encode_4d_bf16(enc, &tm_v, v, dk, bk))
            return MLA_ERR_CUDA;
    }
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    mla::MainArgs a;
    std::memset(&a, 0, sizeof a);
    a.seqlens = seqlens;
    a.B = pl.B;
    a.R = R;
    a.L_max = pl.L_max;
    a.P = pl.num_partitions;
    a.NG = pl.num_groups;
    a.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634074);
    a.out = static_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.part_o = reinterpret_cast<float*>(ws + lay.part_o_off);
    a.part_lse = reinterpret_cast<float*>(ws + lay.part_lse_off);
    a.status = reinterpret_cast<uint32_t*>(ws);
    const unsigned long long tmo = g_timeout_ns.load();
    a.timeout_ns = tmo ? tmo : kDefaultTimeoutNs;
    a.stall_unit = g_stall_unit.load();
    a.prefetch_tiles = 0;
    a.sinks = sinks;
    a.H = pl.H;
    a.split_tiles = pl.split_tiles;
    a.Sq = pl.Sq;
    a.Hkv = pl.Hkv;
    a.o_scale = 1.f;
    a.q = static_cast<const __nv_bfloat16*>(q);
    if (phases & 1) {
        const mla_status st = (G == 16) ? launch_transposed<16, mla::MhaShape>(pl, tm_q, tm_k, tm_v, a, stream)
                                        : launch_transposed<32, mla::MhaShape>(pl, tm_q, tm_k, tm_v, a, stream);
        if (st != MLA_OK) {
            cudaGetLastError();
            return st;
        }
    }
    if (!(phases & 2)) return MLA_OK;
    mla::CombineArgs c;
    std::memset(&c, 0, sizeof c);
    c.seqlens = seqlens;
    c.B = pl.B;
    c.R = R;
    c.L_max = pl.L_max;
    c.P = pl.num_partitions;
    c.out = a.out;
    c.lse = lse;
    c.part_o = a.part_o;
    c.part_lse = a.part_lse;
    c.sinks = sinks;
    c.H = pl.H;
    c.split_tiles = pl.split_tiles;
    const dim3 cgrid(static_cast<unsigned>(pl.B), static_cast<unsigned>(mla::combine_grid_y(pl.B, R, pl.num_sms)));
    return launch_combine<kMhaD>(cgrid, c, stream);
}

}  // namespace

extern "C" {

mla_status mha_decode_run(const mla_plan* plan, const void* q, const void* k, const void* v, const int32_t* seqlens,
                          float softmax_scale, const float* sinks, void* out, float* lse, void* workspace,
                          size_t workspace_bytes, void* stream) {
    return mha_run_phases(plan, q, k, v, seqlens, softmax_scale, sinks, out, lse, workspace, workspace_bytes, stream,
                          3);
}

mla_status mha_decode_run_phase(const mla_plan* plan, const void* q, const void* k, const void* v,
                                const int32_t* seqlens, float softmax_scale, const float* sinks, void* out, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream, int32_t phase) {
    if (phase != 1 && phase != 2) return MLA_ERR_INVALID_ARG;
    return mha_run_phases(plan, q, k, v, seqlens, softmax_scale, sinks, out, lse, workspace, workspace_bytes, stream,
                          phase);
}

}  // extern "C"
