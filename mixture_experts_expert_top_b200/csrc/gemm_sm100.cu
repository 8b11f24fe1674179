// gemm_sm100.cu -- grouped GEMMs of the MoE layer on sm_100a tensor cores.
//
// What they compute (InfiniLM PR #500 Qwen3-MoE report, §2.2 step 2: one
// grouped GEMM call covers every expert's slab of permuted rows):
//   gate/up:  act[r, i] = bf16( silu(g) * u ),  g = a[r] . W_gu[e, i],
//             u = a[r] . W_gu[e, I + i]   (fp32 accumulation, SwiGLU fused)
//   down:     y[r, h]  = bf16( act[r] . W_d[e, h] )
// for every permuted row r of expert e (offsets[e] <= r < offsets[e+1]).
//
// Design (sm_100a; the FlashInfer PR #7196 analysis §2 describes the same
// operand roles for its W4A16 kernel):
//  - Weights are the MMA's A operand (M = 128 weight rows per tile), tokens
//    are the B operand (N = tokens). The MMA's N is chosen per tile at run
//    time as the routed-token count rounded up to 16, so a decode tile with 5
//    tokens issues N = 16 instructions and reads only 16 token rows.
//  - gate/up tiles hold 128 gate rows and the matching 128 up rows: two MMAs
//    per K step into two TMEM accumulators, so each epilogue thread finds g
//    and u of the same (feature, token) in the same TMEM lane.
//  - Persistent CTAs (one per SM) walk a static list of (expert, feature
//    block, token block) tiles; experts with no tokens have no tiles.
//  - Warp roles: warp 0 issues TMA loads into a STAGES-deep shared-memory
//    ring, warp 1 issues tcgen05.mma (one thread) and owns the TMEM
//    allocation, warps 2-5 drain the double-buffered TMEM accumulators
//    (tcgen05.ld), apply SwiGLU and store bf16 rows.
//  - W4A16 (INT4 = true): the TMA brings packed int4 weight tiles; warps 2-5
//    first turn each stage into a swizzled bf16 tile in shared memory
//    (w = bf16(q * scale)), then the MMA reads it like a bf16 tile; the same
//    warps run the epilogue once a tile's K loop is converted.
//  - Every wait is bounded (see mbar_wait); a timeout raises the device flag
//    and unwinds the CTA.
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kBM = 128;          // weight rows per tile (MMA M)
constexpr int kBK = 64;           // K elements per stage (one 128-byte swizzle row)
constexpr int kBoxN = 16;         // token rows per TMA box
constexpr int kThreads = 192;     // 6 warps
constexpr int kTileBytesA = kBM * kBK * 2;          // 16 KB bf16 tile
constexpr int kPackedBytesA = kBM * kBK / 2;        // 4 KB int4 tile
constexpr int kMaxExperts = 1024;

template <int BN, int STAGES, bool SWIGLU, bool INT4>
struct Cfg {
    static constexpr int kNumA = SWIGLU ? 2 : 1;
    static constexpr int kBBytes = BN * kBK * 2;
    static constexpr int kStageBytes = kNumA * kTileBytesA + kBBytes;
    static constexpr int kPackedStage = INT4 ? kNumA * kPackedBytesA : 0;
    static constexpr int kAccCols = SWIGLU ? 2 * BN : BN;
    static constexpr int kTmemCols = (2 * kAccCols <= 32) ? 32 : (2 * kAccCols <= 64) ? 64
                                   : (2 * kAccCols <= 128) ? 128 : (2 * kAccCols <= 256) ? 256 : 512;
    // ring, then packed ring (int4), then barriers and bookkeeping
    static constexpr int kRingBytes = STAGES * kStageBytes;
    static constexpr int kPackedRingBytes = STAGES * kPackedStage;
    static constexpr int kBarBytes = 8 * (4 * STAGES + 4 + 1);
    static constexpr int kMiscBytes = 64 + 2 * (kMaxExperts + 1) * 4;
    static constexpr int kSmemBytes = 1024 /*align slack*/ + kRingBytes + kPackedRingBytes + kBarBytes + kMiscBytes;
    static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(2 * kAccCols <= 512, "TMEM holds 512 fp32 columns");
    static_assert(BN % kBoxN == 0 && BN <= 256, "BN");
};

struct Params {
    const int32_t *offsets;
    int E, K, m_out, w_rows, P;
    uint16_t *out;
    int *err;
    const uint16_t *w_scales;   // int4: [E * w_rows, K/128]
    int evict_first_weights;
};

// Tile bookkeeping shared by the three roles.
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

// W4A16 decoding of one 16-byte packed chunk (32 int4 values of one row) into
// four 16-byte bf16 chunks: w = bf16_rne(q * scale). The fp32 product is exact
// (q has at most 4 significant bits, the bf16 scale 8), so converting it with
// round-to-nearest-even is the only rounding.
__device__ __forceinline__ void dequant32(const uint4 &packed, float scale, uint4 (&o)[4]) {
    const uint32_t words[4] = {packed.x, packed.y, packed.z, packed.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
        const uint32_t x = words[wi];
        uint32_t r[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const uint32_t byte = (x >> (8 * b)) & 0xFFu;
            const int lo = static_cast<int>((byte & 0xFu) ^ 8u) - 8;     // sign-extended low nibble
            const int hi = static_cast<int>((byte >> 4) ^ 8u) - 8;
            const __nv_bfloat162 v = __floats2bfloat162_rn(static_cast<float>(lo) * scale,
                                                           static_cast<float>(hi) * scale);
            r[b] = *reinterpret_cast<const uint32_t *>(&v);
        }
        o[wi] = make_uint4(r[0], r[1], r[2], r[3]);
    }
}

template <int BN, int STAGES, bool SWIGLU, bool INT4>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Params p) {
    using C = Cfg<BN, STAGES, SWIGLU, INT4>;
    extern __shared__ uint8_t smem_raw[];
    // operand tiles need 1024-byte alignment in the shared window (swizzle atoms)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = smem;                                    // STAGES x [A0 | A1 | B]
    uint8_t *pring = smem + C::kRingBytes;                   // int4: STAGES x [Aq0 | Aq1]
    uint64_t *bars = reinterpret_cast<uint64_t *>(pring + C::kPackedRingBytes);
    uint64_t *full_bar = bars;                 // TMA -> (converter | MMA)
    uint64_t *empty_bar = bars + STAGES;       // MMA -> TMA
    uint64_t *conv_bar = bars + 2 * STAGES;    // converter -> MMA (int4)
    uint64_t *tfull_bar = bars + 3 * STAGES;   // MMA -> epilogue, 2 buffers
    uint64_t *tempty_bar = tfull_bar + 2;      // epilogue -> MMA, 2 buffers
    uint64_t *drain_bar = tempty_bar + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int *off_s = reinterpret_cast<int *>(tmem_holder + 16);  // [E+1]
    int *pre_s = off_s + (kMaxExperts + 1);                  // [E+1] tile prefix

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = p.E;
    const int MB = (p.m_out + kBM - 1) / kBM;
    const int KB = (p.K + kBK - 1) / kBK;

    // ---- prologue: barriers, TMEM, tile prefix --------------------------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
            mbar_init(&conv_bar[s], 128);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 128);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::kTmemCols);
        tmem_relinquish();
    }
    for (int i = threadIdx.x; i <= E; i += kThreads) off_s[i] = __ldg(p.offsets + i);
    __syncthreads();
    // tiles per expert, then an inclusive scan by segments of ceil((E)/192)
    {
        const int seg = (E + kThreads - 1) / kThreads;
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
        // exclusive scan of segment totals over the 192 threads
        __shared__ int wsum[kThreads / 32];
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
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    const int total_tiles = pre_s[E];

    if (warp == 0) {
        // ================================ TMA producer ==========================
        if (lane == 0) {
            const uint64_t pol_w = p.evict_first_weights ? l2_policy_evict_first() : l2_policy_evict_last();
            const uint64_t pol_x = l2_policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
                const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
                const int nbox = ti.n_mma / kBoxN;
                const int a_row = ti.e * p.w_rows + ti.mb * kBM;
                const uint32_t a_bytes = INT4 ? C::kNumA * kPackedBytesA : C::kNumA * kTileBytesA;
                const uint32_t tx = a_bytes + nbox * kBoxN * kBK * 2;
                bool ok = true;
                for (int kb = 0; kb < KB && ok; ++kb) {
                    ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.err);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&full_bar[stage], tx);
                    uint8_t *st = ring + stage * C::kStageBytes;
                    if (INT4) {
                        uint8_t *pq = pring + stage * C::kPackedStage;
                        tma_load_2d(pq, &tmA, &full_bar[stage], kb * (kBK / 2), a_row, pol_w);
                        if (SWIGLU)
                            tma_load_2d(pq + kPackedBytesA, &tmA, &full_bar[stage], kb * (kBK / 2), a_row + p.m_out,
                                        pol_w);
                    } else {
                        tma_load_2d(st, &tmA, &full_bar[stage], kb * kBK, a_row, pol_w);
                        if (SWIGLU)
                            tma_load_2d(st + kTileBytesA, &tmA, &full_bar[stage], kb * kBK, a_row + p.m_out, pol_w);
                    }
                    uint8_t *sb = st + C::kNumA * kTileBytesA;
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(sb + b * kBoxN * kBK * 2, &tmB, &full_bar[stage], kb * kBK, ti.row0 + b * kBoxN,
                                    pol_x);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ============================
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
                const uint32_t idesc = idesc_bf16_f32(kBM, ti.n_mma);
                ok = mbar_wait(&tempty_bar[buf], bphase ^ 1, abort_flag, p.err);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d0 = tmem_base + buf * C::kAccCols;
                for (int kb = 0; kb < KB; ++kb) {
                    ok = mbar_wait(INT4 ? &conv_bar[stage] : &full_bar[stage], phase, abort_flag, p.err);
                    if (!ok) break;
                    tc_fence_after_sync();
                    const uint32_t st = smem_u32(ring + stage * C::kStageBytes);
                    const uint64_t da0 = sw128_kmajor_desc(st);
                    const uint64_t da1 = sw128_kmajor_desc(st + kTileBytesA);
                    const uint64_t db = sw128_kmajor_desc(st + C::kNumA * kTileBytesA);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k) {
                        const uint32_t acc = (kb | k) != 0;
                        // +32 bytes per K step inside the swizzled row: +2 in the >>4 address field
                        umma_bf16_ss(d0, da0 + 2 * k, db + 2 * k, idesc, acc);
                        if (SWIGLU) umma_bf16_ss(d0 + BN, da1 + 2 * k, db + 2 * k, idesc, acc);
                    }
                    umma_commit(&empty_bar[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(&tfull_bar[buf]);
                if (++buf == 2) { buf = 0; bphase ^= 1; }
            }
            // all issued MMAs complete before TMEM is released
            umma_commit(drain_bar);
            volatile int never = 0;
            mbar_wait(drain_bar, 0, &never, p.err);
        }
    } else {
        // ============ warps 2-5: int4 converters, then the epilogue =============
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int et = threadIdx.x - 64;        // 0..127
        int stage = 0;
        uint32_t phase = 0;
        int buf = 0;
        uint32_t bphase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
            if (INT4) {
                const int a_row = ti.e * p.w_rows + ti.mb * kBM + et;
                const int srows = p.E * p.w_rows;
                const int kgroups = p.K / 128;
                for (int kb = 0; kb < KB; ++kb) {
                    ok = mbar_wait(&full_bar[stage], phase, abort_flag, p.err);
                    if (!ok) break;
                    const uint8_t *pq = pring + stage * C::kPackedStage;
                    uint8_t *st = ring + stage * C::kStageBytes;
#pragma unroll
                    for (int a = 0; a < C::kNumA; ++a) {
                        const int row = a_row + a * p.m_out;
                        const float scale =
                            row < srows ? bf16_bits_to_float(__ldg(p.w_scales + static_cast<size_t>(row) * kgroups +
                                                                    (kb * kBK) / 128))
                                        : 0.f;
                        const uint4 *src = reinterpret_cast<const uint4 *>(pq + a * kPackedBytesA + et * (kBK / 2));
                        uint8_t *dst_row = st + a * kTileBytesA + et * 128;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            uint4 o[4];
                            dequant32(src[half], scale, o);
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const int chunk = half * 4 + c;
                                *reinterpret_cast<uint4 *>(dst_row + ((chunk ^ (et & 7)) << 4)) = o[c];
                            }
                        }
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(&conv_bar[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            ok = mbar_wait(&tfull_bar[buf], bphase, abort_flag, p.err);
            if (!ok) break;
            tc_fence_after_sync();
            const int f = ti.mb * kBM + q * 32 + lane;         // output feature of this thread
            const bool f_ok = f < p.m_out;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * C::kAccCols;
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

    __syncthreads();
    if (*abort_flag) {
        // let copies already in flight land before the CTA's memory is reused
        for (int i = 0; i < 1000; ++i) __nanosleep(1000);
    }
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes, uint64_t cols,
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

int num_sms() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

template <int BN, int STAGES, bool SWIGLU, bool INT4>
cudaError_t run(const GemmArgs &g, cudaStream_t s) {
    using C = Cfg<BN, STAGES, SWIGLU, INT4>;
    CUtensorMap ta, tb;
    const uint64_t a_rows = static_cast<uint64_t>(g.E) * g.w_rows;
    bool ok;
    if (INT4)
        ok = make_map(&ta, g.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, g.K / 2, a_rows, kBK / 2, kBM,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    else
        ok = make_map(&ta, g.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.K, a_rows, kBK, kBM,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&tb, g.a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.K, g.P, kBK, kBoxN,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    Params p;
    p.offsets = g.offsets;
    p.E = g.E;
    p.K = g.K;
    p.m_out = g.m_out;
    p.w_rows = g.w_rows;
    p.P = g.P;
    p.out = g.out;
    p.err = g.err;
    p.w_scales = g.w_scales;
    p.evict_first_weights = BN <= 32;
    auto kern = grouped_gemm_kernel<BN, STAGES, SWIGLU, INT4>;
    cudaError_t st = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (st != cudaSuccess) return st;
    const long long MB = (g.m_out + kBM - 1) / kBM;
    const long long max_tiles = ((static_cast<long long>(g.P) + BN - 1) / BN + std::min(g.E, g.P)) * MB;
    const int grid = static_cast<int>(std::min<long long>(num_sms(), max_tiles));
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, kThreads, C::kSmemBytes, s>>>(ta, tb, p);
    return cudaGetLastError();
}

template <bool SWIGLU, bool INT4>
cudaError_t dispatch_bn(const GemmArgs &g, cudaStream_t s) {
    const double avg = static_cast<double>(g.P) / g.E;   // pairs per expert if the load were even
    if (SWIGLU) {
        if (avg <= 24) return run<32, INT4 ? 4 : 6, SWIGLU, INT4>(g, s);
        if (avg <= 48) return run<64, INT4 ? 4 : 5, SWIGLU, INT4>(g, s);
        return run<128, INT4 ? 3 : 4, SWIGLU, INT4>(g, s);
    } else {
        if (avg <= 24) return run<32, INT4 ? 8 : 10, SWIGLU, INT4>(g, s);
        if (avg <= 48) return run<64, INT4 ? 6 : 8, SWIGLU, INT4>(g, s);
        return run<128, INT4 ? 5 : 6, SWIGLU, INT4>(g, s);
    }
}

// Standalone W4A16 decoding (same arithmetic as the GEMMs' converter warps).
__global__ void dequant_int4_kernel(const uint4 *__restrict__ q, const uint16_t *__restrict__ scales, int rows,
                                    int K, uint4 *__restrict__ out) {
    const long long chunks_per_row = K / 32;   // 16 packed bytes = 32 values
    const long long total = static_cast<long long>(rows) * chunks_per_row;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long r = i / chunks_per_row;
        const int c = static_cast<int>(i - r * chunks_per_row);
        const float scale = bf16_bits_to_float(__ldg(scales + r * (K / 128) + (c * 32) / 128));
        uint4 o[4];
        dequant32(__ldg(q + i), scale, o);
#pragma unroll
        for (int j = 0; j < 4; ++j) out[i * 4 + j] = o[j];
    }
}

}  // namespace

cudaError_t launch_grouped_gemm(const GemmArgs &g, cudaStream_t s) {
    if (g.P == 0) return cudaSuccess;
    if (g.fmt == 0) return g.swiglu ? dispatch_bn<true, false>(g, s) : dispatch_bn<false, false>(g, s);
    return g.swiglu ? dispatch_bn<true, true>(g, s) : dispatch_bn<false, true>(g, s);
}

cudaError_t launch_dequant_int4(const uint8_t *q, const uint16_t *scales, int rows, int K, uint16_t *out,
                                cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const long long total = static_cast<long long>(rows) * (K / 32);
    long long blocks = (total + 255) / 256;
    if (blocks > 148LL * 16) blocks = 148LL * 16;
    dequant_int4_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(reinterpret_cast<const uint4 *>(q), scales, rows,
                                                                  K, reinterpret_cast<uint4 *>(out));
    return cudaGetLastError();
}

}  // namespace moe
