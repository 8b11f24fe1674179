// gemm_common.cuh -- pieces shared by the grouped-GEMM kernels of
// libmoe_b200 (gemm_sm100.cu: weights on the MMA's M side, for few tokens
// per expert; gemm_prefill_sm100.cu: tokens on the M side, for many):
// constants, kernel parameters, the per-expert tile list, the epilogue of the
// weights-on-M kernels and the host-side tensor-map helpers.
#pragma once

#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace gemm {

constexpr int kBM = 128;          // weight rows per tile (MMA M)
constexpr int kBK = 64;           // K elements per bf16 stage / per int4 quarter (one 128-byte bf16 row)
constexpr int kBoxN = 16;         // token rows per TMA box
constexpr int kTileBytesA = kBM * kBK * 2;          // 16 KB bf16 tile (128 x 64)
constexpr int kBoxBytesB = kBoxN * kBK * 2;         // 2 KB token box (16 x 64)
constexpr int kMaxExperts = 1024;
constexpr int kSmemLimit = 232448;                  // 227 KB per CTA
constexpr int kEpiThreads = 128;                    // warps 2-5

// int4 kernel (gemm_sm100.cu)
constexpr int kQuarters = 4;                        // 64-K quarters per int4 stage (K = 256)
constexpr int kPackedTile = kBM * 128;              // 16 KB: 128 rows x 128 packed bytes
constexpr int kConvGroups = kQuarters;              // 4 x 4 decode warps: one set of 4 per quarter
constexpr int kMaxTmemA = 8;
constexpr int kGuessKBlocks = 8;                    // weight K-blocks prefetched on a guess

struct Params {
    const int32_t *offsets;
    const int32_t *perm;        // token operand gathered through perm (nullptr: rows in permuted order)
    int top_k;
    int E, K, m_out, w_rows, P;
    uint16_t *out;
    int *err;
    const uint16_t *w_scales;   // int4: [E * w_rows, K/128]
    int evict_first_weights;
    int hints;                  // kGemmHint* bits
    const uint16_t *a;          // the token operand's rows (GemmArgs::a), for kernels that copy them without TMA
};

// W4A16 decoding of one 32-bit word of packed int4 (K elements 8i..8i+7 of a
// row; byte b holds element 2b in its low nibble, 2b+1 in its high nibble,
// two's complement) into four bf16x2 words (elements 2j, 2j+1 in word j):
//   w = bf16_rne(q * scale)
// Each nibble pair is placed in the mantissas of a bf16x2 with exponent 2^7
// and biased to n = q + 8 (the bias is the flip of the nibble's sign bit,
// folded into the same three-input logic op), giving bf16 (128 + n) exactly;
// subtracting 136 gives q exactly, and one bf16 multiply by the scale rounds
// the exact product once, to nearest even.
__device__ __forceinline__ void dequant_word(uint32_t packed, __nv_bfloat162 scale2, uint32_t *out4) {
    const uint32_t hi = packed >> 4;                       // odd elements move to the low nibble of each byte
    const __nv_bfloat162 bias = __floats2bfloat162_rn(136.0f, 136.0f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // byte 0 <- element 2j (low nibble of byte j), byte 2 <- element 2j+1
        const uint32_t r = __byte_perm(packed, hi, static_cast<uint32_t>(j | ((4 + j) << 8)));
        // bits of 0x000F000F: r ^ 0x00080008 (n = q + 8); other bits: 0x43004300
        const uint32_t v = (r & 0x000F000Fu) ^ 0x43084308u;
        const __nv_bfloat162 q = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&v), bias);
        const __nv_bfloat162 w = __hmul2(q, scale2);
        out4[j] = *reinterpret_cast<const uint32_t *>(&w);
    }
}

__device__ __forceinline__ __nv_bfloat162 bf16_pair(uint16_t bits) {
    const __nv_bfloat16 b = __ushort_as_bfloat16(bits);
    return __halves2bfloat162(b, b);
}

// Tile bookkeeping shared by the roles.
struct TileInfo {
    int e, mb, row0, valid, n_mma;
};

__device__ __forceinline__ TileInfo decode_tile(int tile, const int *pre, const int *off, int E, int MB, int BN) {
    int lo = 0, hi = E - 1;             // largest e with pre[e] <= tile (never an empty expert)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    TileInfo t;
    t.e = lo;
    const int local = tile - pre[lo];
    t.mb = local % MB;
    const int nb = local / MB;
    t.row0 = off[lo] + nb * BN;
    const int cnt = off[lo + 1] - off[lo];
    t.valid = min(BN, cnt - nb * BN);
    t.n_mma = (t.valid + 15) & ~15;
    return t;
}

// Row of the token operand's tensor for permuted row r: perm[r] / top_k in
// gather mode (rows past P read row 0; they are never stored), else r.
__device__ __forceinline__ int token_row(const Params &p, int r) {
    if (!p.perm) return r;
    if (r >= p.P) return 0;
    int v = __ldg(p.perm + r);
    if (kDebugBounds && (v < 0 || v >= p.P)) {
        raise_error(p.err, kErrBounds);
        v = 0;
    }
    return v / p.top_k;
}

// Copies offsets into shared memory and builds pre[e] = number of tiles of
// experts 0..e-1 (a block-wide scan). All threads of the CTA call it.
template <int NT>
__device__ __forceinline__ void build_tile_prefix(const int32_t *offsets, int E, int MB, int BN, int *off_s,
                                                  int *pre_s, int P = 0, int *err = nullptr) {
    __shared__ int wsum[NT / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // L2 reads (no L1 line can be stale): a kernel launched with an early
    // start may read offsets before griddepcontrol.wait (kGemmHintOffsetsReady)
    for (int i = threadIdx.x; i <= E; i += NT) off_s[i] = __ldcg(offsets + i);
    __syncthreads();
    if (kDebugBounds && threadIdx.x == 0) {
        // offsets must start at 0, never decrease and end at P
        bool bad = off_s[0] != 0 || off_s[E] != P;
        int prev = 0;
        for (int i = 0; i <= E; ++i) {
            const int v = min(max(off_s[i], prev), P);
            bad |= v != off_s[i];
            off_s[i] = v;
            prev = v;
        }
        off_s[0] = 0;
        if (bad) raise_error(err, kErrBounds);
    }
    if (kDebugBounds) __syncthreads();
    const int seg = (E + NT - 1) / NT;
    const int b0 = threadIdx.x * seg;
    int local = 0;
    for (int i = 0; i < seg; ++i) {
        const int e = b0 + i;
        if (e < E) {
            const int cnt = off_s[e + 1] - off_s[e];
            local += ((cnt + BN - 1) / BN) * MB;
            pre_s[e + 1] = local;        // segment-local inclusive
        }
    }
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int before = x - local;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    for (int i = 0; i < seg; ++i) {
        const int e = b0 + i;
        if (e < E) pre_s[e + 1] += before;
    }
    if (threadIdx.x == 0) pre_s[0] = 0;
}

// Epilogue of warps 2-5: per tile, wait for the accumulator buffer, read it
// with tcgen05.ld (warp w reads TMEM lanes 32*(w%4)...), apply SwiGLU for
// gate/up, round to bf16 and store; then hand the buffer back.
template <int BN, bool SWIGLU, int ACC_COLS>
__device__ __forceinline__ void run_epilogue(const Params &p, const int *pre_s, const int *off_s, int total_tiles,
                                             int MB, uint32_t tmem_base, uint64_t *tfull_bar, uint64_t *tempty_bar,
                                             volatile int *abort_flag, uint32_t max_sleep_ns = 512) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    int buf = 0;
    uint32_t bphase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
        const TileInfo ti = decode_tile(tile, pre_s, off_s, p.E, MB, BN);
        if (!mbar_wait(&tfull_bar[buf], bphase, abort_flag, p.err, max_sleep_ns)) break;
        tc_fence_after_sync();
        const int f = ti.mb * kBM + q * 32 + lane;         // output feature of this thread
        const bool f_ok = f < p.m_out;
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * ACC_COLS;
        for (int c0 = 0; c0 < ti.n_mma; c0 += 16) {
            uint32_t g[16], u[16];
            tmem_ld_32x32b_x16(tb + c0, g);
            if (SWIGLU) tmem_ld_32x32b_x16(tb + BN + c0, u);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int n = c0 + j;
                if (f_ok && n < ti.valid) {
                    float v = __uint_as_float(g[j]);
                    if (SWIGLU) {
                        const float uu = __uint_as_float(u[j]);
                        v = v / (1.0f + expf(-v)) * uu;
                    }
                    const __nv_bfloat16 bv = __float2bfloat16_rn(v);
                    p.out[static_cast<size_t>(ti.row0 + n) * p.m_out + f] = __bfloat16_as_ushort(bv);
                }
            }
        }
        tc_fence_before_sync();
        mbar_arrive(&tempty_bar[buf]);
        if (++buf == 2) { buf = 0; bphase ^= 1; }
    }
}


// ------------------------------------------------------------------ host side

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D row-major map: `cols` contiguous elements per row, `rows` rows.
inline bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes, uint64_t cols,
              uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same with an explicit row pitch in bytes (for packed 4-bit elements,
// whose rows are cols / 2 bytes).
inline bool make_map_pitched(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows,
                             uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map of the token operand: a [rows, K] bf16 with the 128-byte
// swizzle; a box of box_rows rows, or of one row for gather4 loads.
inline bool make_token_map(CUtensorMap *m, const GemmArgs &g, uint32_t box_rows) {
    const uint64_t rows = g.perm ? static_cast<uint64_t>(g.T) : static_cast<uint64_t>(g.P);
    return make_map(m, g.a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.K, rows, kBK, g.perm ? 1 : box_rows,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

inline int num_sms() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

inline Params make_params(const GemmArgs &g, int BN) {
    Params p;
    p.offsets = g.offsets;
    p.perm = g.perm;
    p.a = static_cast<const uint16_t *>(g.a);
    p.top_k = g.top_k;
    p.E = g.E;
    p.K = g.K;
    p.m_out = g.m_out;
    p.w_rows = g.w_rows;
    p.P = g.P;
    p.out = g.out;
    p.err = g.err;
    p.w_scales = g.w_scales;
    p.evict_first_weights = BN <= 32;
    p.hints = g.hints;
    return p;
}

inline int grid_for(const GemmArgs &g, int BN) {
    const long long MB = (g.m_out + kBM - 1) / kBM;
    const long long max_tiles = ((static_cast<long long>(g.P) + BN - 1) / BN + std::min(g.E, g.P)) * MB;
    return static_cast<int>(std::min<long long>(num_sms(), max_tiles));
}

}  // namespace gemm
}  // namespace moe
