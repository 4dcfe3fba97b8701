// Grouped 8-bit GEMMs on the 5th-generation tensor cores (tcgen05: kind::i8
// for INT8 experts with INT32 accumulators, kind::f8f6f4 for E4M3 experts with
// fp32 accumulators; "Day0 adaptation of ultra-large model inference",
// section 1: FP8 or INT8 expert layers) for the expert FFN of the W8A8 MoE
// layer ("MiniMax-M3 W8A8 on K100AI",
// s1.2: INT8 x INT8 on the INT8 GEMM path with integer accumulation; s4.3:
// fuse the expert FFN and stay in INT8 between the two matmuls; "Day0
// adaptation of ultra-large model inference", section 4: grouped GEMM over the
// expert-sorted tokens).
//
// One persistent kernel per GEMM, one CTA per SM.  Tiles of 128 sorted rows
// (one expert) x 256 output channels, K in blocks of 128 bytes:
//   warp 0      TMA producer: A tile (128 x 128 B) and B tile (256 x 128 B) per
//               k-block into a 4-stage shared-memory ring (128-byte swizzle)
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               (M=128, N=256, K=32 per instruction) into one of two 256-column
//               INT32 accumulators, double-buffered so the epilogue of one tile
//               runs under the main loop of the next
//   warps 2..9  epilogue: tcgen05.ld of their 32-lane quarter of the
//               accumulator, dequantisation and the fused math, global stores
// GEMM1 epilogue: g, u dequantised (per-token x per-channel scales), h = silu(g)
// u written in fp32 with one partial row maximum per 64 columns; the row-wide
// INT8 requantisation of h (max over all f channels) is a separate,
// bandwidth-bound kernel (requant_kernel below), so no CTA ever waits for or
// coordinates with another.  GEMM2 epilogue: o = acc2 sh sw w in fp32 per
// sorted row.
// Epilogue stores go through a small swizzled shared-memory buffer per warp so
// that each global store instruction writes whole 128-byte rows.
//
// Every wait on an mbarrier is bounded by the global timer; when a wait runs
// out the kernel records MOE_ERR_TIMEOUT in the status word, stops issuing
// work, waits (bounded) for its copies and MMAs in flight, frees its TMEM and
// returns.
#include <cuda.h>

#include <climits>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK;                  // 16 KB
constexpr int kBBytes = BN * BK;                  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + kEpiWarps * 32;     // 320
constexpr uint32_t kTmemCols = 2 * BN;            // two 256-column accumulators
constexpr uint64_t kWaitBudgetNs = 2000000000ull; // 2 s per wait
constexpr int kEpiStoreBytes = 16 * 32 * 4;      // 16 rows x 32 fp32 per epilogue warp (store staging)
constexpr int kEpiStageBytes = kEpiStoreBytes + 512;   // + the tile's 128 column scales
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + (size_t)kEpiWarps * kEpiStageBytes + 1024 + 256;


// Instruction descriptors (both operands K-major, N>>3 at bit 17, M>>4 at bit 24):
//   kind::i8     D = s32 (bits 4-5 = 2), A and B signed 8-bit (bits 7-9, 10-12 = 1)
//   kind::f8f6f4 D = f32 (bits 4-5 = 1), A and B E4M3 (bits 7-9, 10-12 = 0)
template <int FMT, int M = BM, int N = BN>
__host__ __device__ constexpr uint32_t idesc() {
    return (FMT == FMT_E4M3 ? (1u << 4) : ((2u << 4) | (1u << 7) | (1u << 10))) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// Row of the tiled weight copy at which k-block kb of the weight rows
// starting at brow (a multiple of 128) begins: [row tile][k-block][256 rows].
__device__ __forceinline__ int tiled_row(int brow, int kb, int nkb) {
    return ((brow / BN) * nkb + kb) * BN + brow % BN;
}

template <int NS>
struct CtlT {
    uint64_t full[NS];
    uint64_t empty[NS];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
using Ctl = CtlT<kStages>;

struct TcParams {
    int N, K, n_tiles_n, f, k;
    const int32_t* meta;
    const int32_t* tiles;     // [m-tile][2] = (expert, first row)
    const int32_t* pairs;     // [pair tile][2] = (expert, first of 256 rows), for CTA pairs
    const int32_t* offsets;   // [E+1]
    const int32_t* row2ts;
    const float* topk_w;
    const float* sx;          // GEMM1: per-token activation scale
    const float* sw0;         // GEMM1: sw_gate [E][f]; GEMM2: sw_dn [E][d]
    const float* sw1;         // GEMM1: sw_up [E][f]
    const float* sh;          // GEMM2: per-row h scale
    float* h32;               // GEMM1: h [rows][f]
    float* pamax;             // GEMM1: per-row partial max [rows][f/64]
    void* o;                  // GEMM2: [rows][d], fp32 or (o_bf16) bf16
    int o_bf16;               // GEMM2: per-slot rows in bf16 (bf16-output layers)
    int tma_c;                // the kernel's output map (tm_c) serves bulk tensor stores of full 32-row
                              // chunks (64-byte rows: GEMM1 16 fp32 h values, GEMM2 32 bf16 values)
    int32_t* acc_dbg;         // optional raw accumulators (canonical channel order)
    int32_t* status;
};

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for the phase of parity `parity` to complete.  Returns false
// (after recording the timeout) when the budget runs out or another role
// already gave up.
// Record a timeout: status[0] = MOE_ERR_TIMEOUT; the first reporter also
// leaves where it gave up in status[1..4] (site, block, tile iteration, extra).
__device__ void report_timeout(int32_t* status, int site, int iter, int extra) {
    atomicExch(status, (int32_t)MOE_ERR_TIMEOUT);
    if (atomicCAS(status + 1, 0, site) == 0) {
        status[2] = (int32_t)blockIdx.x;
        status[3] = iter;
        status[4] = extra;
    }
}

__device__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int32_t* status,
                          int site = 0, int iter = 0) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (global_timer() - t0 > kWaitBudgetNs) {
            *abort = 1;
            report_timeout(status, site, iter, (int)parity);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// TMA store of a staged box from this CTA's shared memory (bulk async group);
// the staged data must have been made visible to the async proxy
// (fence.proxy.async.shared::cta by the writing threads) first.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The previous bulk stores of this thread have finished reading shared memory.
__device__ __forceinline__ void tma_store_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// The previous bulk stores of this thread are complete.
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row atoms of
// 1024 bytes (stride byte offset 1024); leading byte offset unused for this
// layout; descriptor version 1 (bit 46); layout type 2 = SWIZZLE_128B.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// One K=32 MMA of 8-bit operands, M x N = 128 x 256 unless the instruction
// descriptor ID says otherwise: INT8 (s32 accumulators) or E4M3 (f32
// accumulators).
template <int FMT, uint32_t ID = idesc<FMT>()>
__device__ __forceinline__ void mma_8bit(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accum) {
    if (FMT == FMT_E4M3)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
            "l"(adesc), "l"(bdesc), "r"(ID), "r"(accum));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
            "l"(adesc), "l"(bdesc), "r"(ID), "r"(accum));
}

// Accumulator word as a float: INT32 converted, fp32 reinterpreted.
template <int FMT>
__device__ __forceinline__ float acc_value(uint32_t a) {
    return FMT == FMT_E4M3 ? __uint_as_float(a) : __int2float_rn((int)a);
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ epilogues

enum { EPI_SWIGLU = 0, EPI_DOWN = 1 };

// Store a warp's 32 rows x 32 fp32 values (lane l holds row l's values v[0..31])
// to rows gbase + l*ld (only the first nvalid rows), coalesced: two passes of 16
// rows through a 2 KB buffer whose 16-byte chunks are XOR-swizzled by row, so
// neither the shared-memory writes nor the reads conflict.
__device__ __forceinline__ void store_rows32(float* stage, const uint32_t (&v)[32], float* gbase,
                                             int64_t ld, int nvalid, int lane) {
    float4* st4 = reinterpret_cast<float4*>(stage);
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
        if ((lane >> 4) == pass) {
            const int r = lane & 15;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                st4[r * 8 + (j ^ (r & 7))] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                         __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int r = it * 4 + (lane >> 3), c = lane & 7;
            const float4 q = st4[r * 8 + (c ^ (r & 7))];
            const int row = pass * 16 + r;
            if (row < nvalid) reinterpret_cast<float4*>(gbase + (int64_t)row * ld)[c] = q;
        }
        __syncwarp();
    }
}

// Release of an accumulator buffer by one epilogue warp: a local arrive, or,
// for a CTA pair, an arrive on the pair leader's barrier (same offset in the
// leader's shared memory), which counts the warps of both CTAs.  Only the
// warp's tensor-memory reads must precede it (tcgen05.wait::ld and the
// before-thread-sync fence); the default CTA-scope semantics of the arrive do
// not make it wait for the warp's outstanding global stores.
template <bool PAIR>
__device__ __forceinline__ void release_acc(uint64_t* bar) {
    if (PAIR) {
        uint32_t remote;
        asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(remote) : "r"(smem_u32(bar)));
        asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
    } else {
        mbar_arrive(bar);
    }
}

// The per-tile inputs of an epilogue warp, fetched before it waits for the
// accumulator so that their memory latency overlaps the tile's MMAs: the
// scalars of its lane's row (GEMM1: the token's activation scale; GEMM2: the
// row's h scale and routing weight) into registers, and the 128 column scales
// of its half tile into its slice `sc` of shared memory (GEMM1: 64 gate then
// 64 up scales of its 64 h channels; GEMM2: the scales of its 128 output
// columns), one 16-byte load per lane.
template <int EPI>
__device__ __forceinline__ void epi_prefetch(const TcParams& p, int e, int nt, int half, int grow, bool valid,
                                             float* sc, int lane, float& r0, float& r1) {
    if (EPI == EPI_SWIGLU) {
        const float* base = (lane < 16 ? p.sw0 : p.sw1) + (int64_t)e * p.f + nt * 128 + 64 * half;
        reinterpret_cast<float4*>(sc)[lane] = reinterpret_cast<const float4*>(base)[lane & 15];
        r0 = valid ? p.sx[p.row2ts[grow] / p.k] : 0.0f;
        r1 = 0.0f;
    } else {
        const float* base = p.sw0 + (int64_t)e * p.N + nt * BN + 128 * half;
        reinterpret_cast<float4*>(sc)[lane] = reinterpret_cast<const float4*>(base)[lane];
        r0 = valid ? p.sh[grow] : 0.0f;
        r1 = valid ? p.topk_w[p.row2ts[grow]] : 0.0f;
    }
    __syncwarp();
}

// Store a warp's 32 rows x 64 bytes (lane l holds row l's 16 words w[0..15])
// to the rows [row0, row0 + 32) at column x of a tensor whose map `tmc` has a
// 32-row x 64-byte box with 64-byte swizzle: the rows are staged in that
// layout (16-byte chunks XOR (row / 2) mod 4, the same layout the plain path
// uses) and one lane issues a bulk tensor store, which writes the box
// asynchronously.  When fewer than 32 rows are valid (an expert's last
// rows: the box would overwrite the next expert's) or there is no map, the
// plain stores write the first nvalid rows to gbase.  `stage` is 512-byte
// aligned; before it is rewritten the previous bulk store must have read it.
__device__ __forceinline__ void store_rows_64b(float* stage, const uint32_t (&v)[16], const CUtensorMap* tmc,
                                               int x, int row0, void* gbase, int64_t ld_bytes, int nvalid, int lane) {
    uint4* st4 = reinterpret_cast<uint4*>(stage);
    if (lane == 0) tma_store_wait_read();
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j)
        st4[lane * 4 + (j ^ ((lane >> 1) & 3))] = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    if (tmc && nvalid == 32) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) tma_store_2d(tmc, stage, x, row0);
        return;
    }
    __syncwarp();
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int r = it * 8 + (lane >> 2), c = lane & 3;
        const uint4 q = st4[r * 4 + (c ^ ((r >> 1) & 3))];
        if (r < nvalid) reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(gbase) + (int64_t)r * ld_bytes)[c] = q;
    }
    __syncwarp();
}

// GEMM1 tile: columns 0..127 of the accumulator are gate channels
// nt*128 + c, columns 128..255 the matching up channels.  Each warp owns 32
// rows (its TMEM lane quarter) and 64 of the 128 h columns.  sc, sxt: from
// epi_prefetch<EPI_SWIGLU>.
template <int FMT, bool PAIR = false>
__device__ __forceinline__ void epilogue_swiglu(const TcParams& p, uint32_t taddr, int half, int e,
                                                int nt, int wrow0, int nvalid, float* stage, const float* sc,
                                                float sxt, uint64_t* acc_empty, const CUtensorMap* tmc, int lane) {
    const int f = p.f;
    const bool valid = lane < nvalid;
    const int grow = wrow0 + lane;
    float amax = 0.0f;
    // four 16-column sub-chunks of gate and up words, double-buffered: sub-chunk
    // c + 1 is requested right after sub-chunk c has arrived, so its latency
    // overlaps c's math and stores; the accumulator is released once the last
    // sub-chunk is in registers
    uint32_t gb[2][16], ub[2][16];
    tmem_ld16(taddr + 64 * half, gb[0]);
    tmem_ld16(taddr + 128 + 64 * half, ub[0]);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int col0 = 64 * half + 16 * c;
        uint32_t (&g)[16] = gb[c & 1];
        uint32_t (&u)[16] = ub[c & 1];
        tmem_ld_wait();
        if (c < 3) {
            tmem_ld16(taddr + col0 + 16, gb[(c + 1) & 1]);
            tmem_ld16(taddr + 128 + col0 + 16, ub[(c + 1) & 1]);
        } else {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release_acc<PAIR>(acc_empty);
        }
        const int ch0 = nt * 128 + col0;
        const float* swg = sc + 16 * c;
        const float* swu = sc + 64 + 16 * c;
        if (p.acc_dbg && valid) {
            int32_t* dg = p.acc_dbg + (int64_t)grow * 2 * f + ch0;
            for (int j = 0; j < 16; ++j) {
                dg[j] = (int32_t)g[j];
                dg[f + j] = (int32_t)u[j];
            }
        }
        uint32_t hv[16];
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
            const float4 sg = *reinterpret_cast<const float4*>(swg + j);
            const float4 su = *reinterpret_cast<const float4*>(swu + j);
            const float sgv[4] = {sg.x, sg.y, sg.z, sg.w}, suv[4] = {su.x, su.y, su.z, su.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float gf = __fmul_rn(__fmul_rn(acc_value<FMT>(g[j + q]), sxt), sgv[q]);
                const float uf = __fmul_rn(__fmul_rn(acc_value<FMT>(u[j + q]), sxt), suv[q]);
                const float h = __fmul_rn(moe_silu(gf), uf);
                if (valid) amax = fmaxf(amax, fabsf(h));
                hv[j + q] = __float_as_uint(h);
            }
        }
        store_rows_64b(stage, hv, tmc, ch0, wrow0, p.h32 + (int64_t)wrow0 * f + ch0, (int64_t)f * 4, nvalid, lane);
    }
    if (valid) p.pamax[(int64_t)grow * (f / 64) + nt * 2 + half] = amax;
}

// GEMM2 tile: each warp owns 32 rows and 128 of the 256 output columns.  sc,
// shr, wr: from epi_prefetch<EPI_DOWN>.
template <int FMT, bool PAIR = false>
__device__ __forceinline__ void epilogue_down(const TcParams& p, uint32_t taddr, int half, int e,
                                              int nt, int wrow0, int nvalid, float* stage, const float* sc,
                                              float shr, float wr, uint64_t* acc_empty, const CUtensorMap* tmc,
                                              int lane) {
    const int d = p.N;
    const bool valid = lane < nvalid;
    const int grow = wrow0 + lane;
    // two register sets: chunk c + 1's accumulator words are requested right
    // after chunk c's have arrived, so their latency overlaps chunk c's math
    // and stores
    uint32_t buf2[2][32];
    tmem_ld32(taddr + 128 * half, buf2[0]);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int col0 = 128 * half + 32 * c;
        uint32_t (&a)[32] = buf2[c & 1];
        tmem_ld_wait();
        if (c < 3) {
            tmem_ld32(taddr + col0 + 32, buf2[(c + 1) & 1]);
        } else {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release_acc<PAIR>(acc_empty);
        }
        const int ch0 = nt * BN + col0;
        const float* sw = sc + 32 * c;
        if (p.acc_dbg && valid) {
            int32_t* da = p.acc_dbg + (int64_t)grow * d + ch0;
            for (int j = 0; j < 32; ++j) da[j] = (int32_t)a[j];
        }
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            const float4 s4 = *reinterpret_cast<const float4*>(sw + j);
            const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                a[j + q] = __float_as_uint(
                    __fmul_rn(__fmul_rn(__fmul_rn(acc_value<FMT>(a[j + q]), shr), sv[q]), wr));
        }
        if (p.o_bf16) {
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 16; ++q)
                w[q] = (uint32_t)f32_to_bf16_bits(__uint_as_float(a[2 * q])) |
                       ((uint32_t)f32_to_bf16_bits(__uint_as_float(a[2 * q + 1])) << 16);
            store_rows_64b(stage, w, tmc, ch0, wrow0, reinterpret_cast<uint16_t*>(p.o) + (int64_t)wrow0 * d + ch0,
                           (int64_t)d * 2, nvalid, lane);
        } else
            store_rows32(stage, a, reinterpret_cast<float*>(p.o) + (int64_t)wrow0 * d + ch0, d, nvalid, lane);
    }
}

// Epilogues of the fused launch's swapped-operand plan (at most 32 rows per
// m-tile): the weights are the MMAs' A operand and the tile's token rows the
// B operand (N = 32), so an accumulator holds [weight row][token row]: TMEM
// lane = channel, column = row.  Two accumulators per tile, 32 columns each:
// GEMM1 gate (columns 0..31) and up (32..63) of 128 channels; GEMM2 output
// columns nt*256 + [0, 128) and + [128, 256).  A warp reads its TMEM lane
// quarter (32 channels); per-row scalars are held by lane r and broadcast.
// The arithmetic per element is that of epilogue_swiglu / epilogue_down.
constexpr int kFusedSwapRows = 32;

// GEMM1: warp (quad, half) owns channels nt*128 + 32 quad + lane and rows
// 16 half .. 16 half + 15 (sxr: lane j's row 16 half + j activation scale; sg,
// su: the lane's channel scales).  The partial maximum of each row over the
// warp's 32 channels goes to pamax[row][f / 32].
template <int FMT>
__device__ __forceinline__ void epilogue_swiglu_sw(const TcParams& p, uint32_t taddr, int half, int quad, int nt,
                                                   int row0, int nrows, float sg, float su, float sxr,
                                                   uint64_t* acc_empty, int lane) {
    const int f = p.f;
    const int ch = nt * 128 + 32 * quad + lane;
    const int npart = f / 32, part = nt * 4 + quad;
    uint32_t g[16], u[16];
    tmem_ld16(taddr + 16 * half, g);
    tmem_ld16(taddr + 32 + 16 * half, u);
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acc_empty);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int r = 16 * half + j;
        const float sx = __shfl_sync(0xffffffffu, sxr, j);
        if (r >= nrows) break;   // the same for every lane
        const int64_t grow = row0 + r;
        if (p.acc_dbg) {
            p.acc_dbg[grow * 2 * f + ch] = (int32_t)g[j];
            p.acc_dbg[grow * 2 * f + f + ch] = (int32_t)u[j];
        }
        const float gf = __fmul_rn(__fmul_rn(acc_value<FMT>(g[j]), sx), sg);
        const float uf = __fmul_rn(__fmul_rn(acc_value<FMT>(u[j]), sx), su);
        const float h = __fmul_rn(moe_silu(gf), uf);
        p.h32[grow * f + ch] = h;
        const float m = warp_max(fabsf(h));
        if (lane == 0) p.pamax[grow * npart + part] = m;
    }
}

// GEMM2: warp (quad, half) owns output column nt*256 + 128 half + 32 quad +
// lane for all rows (shr, wr: lane r's row h scale and routing weight; sw: the
// lane's column scale).
template <int FMT>
__device__ __forceinline__ void epilogue_down_sw(const TcParams& p, uint32_t taddr, int half, int quad, int nt,
                                                 int row0, int nrows, float sw, float shr, float wr,
                                                 uint64_t* acc_empty, int lane) {
    const int d = p.N;
    const int col = nt * BN + 128 * half + 32 * quad + lane;
    uint32_t a[32];
    tmem_ld32(taddr + 32 * half, a);
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acc_empty);
#pragma unroll
    for (int r = 0; r < kFusedSwapRows; ++r) {
        const float s_h = __shfl_sync(0xffffffffu, shr, r);
        const float w_r = __shfl_sync(0xffffffffu, wr, r);
        if (r >= nrows) break;   // the same for every lane
        const int64_t grow = row0 + r;
        if (p.acc_dbg) p.acc_dbg[grow * d + col] = (int32_t)a[r];
        const float o = __fmul_rn(__fmul_rn(__fmul_rn(acc_value<FMT>(a[r]), s_h), sw), w_r);
        if (p.o_bf16)
            reinterpret_cast<uint16_t*>(p.o)[grow * d + col] = f32_to_bf16_bits(o);
        else
            reinterpret_cast<float*>(p.o)[grow * d + col] = o;
    }
}

// ------------------------------------------------------------------ the kernel

template <int EPI, int FMT>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_c, const TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    float* epi_stage = reinterpret_cast<float*>(smem + kStages * kStageBytes);
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + kStages * kStageBytes + kEpiWarps * kEpiStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = p.K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], 1);
            mbar_init(&ctl->acc_empty[b], kEpiWarps);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctl->tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    volatile int* abort = &ctl->abort;
    // everything above overlaps the previous kernel; its results are read below
    pdl_wait();
    pdl_trigger();
    const int num_tiles = p.meta[META_NTILES] * p.n_tiles_n;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_par[kStages];
            bool issued[kStages];
            for (int i = 0; i < kStages; ++i) issued[i] = false;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                const int mt = t / p.n_tiles_n, nt = t % p.n_tiles_n;
                const int e = p.tiles[2 * mt], row0 = p.tiles[2 * mt + 1];
                const int brow = e * p.N + nt * BN;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&ctl->empty[s], ph ^ 1, abort, p.status, 1, t)) { ok = false; break; }
                    mbar_arrive_expect_tx(&ctl->full[s], kStageBytes);
                    uint8_t* sa = smem + s * kStageBytes;
                    tma_load_2d(sa, &tm_a, &ctl->full[s], kb * BK, row0);
                    tma_load_2d(sa + kABytes, &tm_b, &ctl->full[s], 0, tiled_row(brow, kb, nkb));
                    issued[s] = true;
                    issued_par[s] = ph;
                    if (++s == kStages) { s = 0; ph ^= 1; }
                }
            }
            // copies in flight land before the CTA ends (bounded)
            for (int i = 0; i < kStages; ++i) {
                if (!issued[i]) continue;
                const uint64_t t0 = global_timer();
                while (!mbar_try_wait(&ctl->full[i], issued_par[i]) && global_timer() - t0 < kWaitBudgetNs) {}
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            int s = 0, buf = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                if (!mbar_wait(&ctl->acc_empty[buf], aph ^ 1, abort, p.status, 2, t)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(buf * BN);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&ctl->full[s], ph, abort, p.status, 3, t)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
                    const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)
                        mma_8bit<FMT>(d_tmem, desc_sw128(a_addr + kk * 32), desc_sw128(b_addr + kk * 32),
                               (kb | kk) != 0 ? 1u : 0u);
                    mma_commit(&ctl->empty[s]);
                    if (++s == kStages) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                mma_commit(&ctl->acc_full[buf]);
                buf ^= 1;
                if (buf == 0) aph ^= 1;
            }
            // all MMAs issued by this thread complete before TMEM is freed (bounded)
            mma_commit(&ctl->drain);
            const uint64_t t0 = global_timer();
            while (!mbar_try_wait(&ctl->drain, 0) && global_timer() - t0 < kWaitBudgetNs) {}
        }
    } else {
        // ---------------- epilogue warps
        const int ew = warp - 2;                 // 0..7
        const int quad = warp & 3;               // TMEM lanes this warp may access
        const int half = ew >> 2;                // which half of the tile's columns
        float* stage = epi_stage + ew * (kEpiStageBytes / 4);
        int buf = 0;
        uint32_t aph = 0;
        float* sc = stage + kEpiStoreBytes / 4;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
            const int mt = t / p.n_tiles_n, nt = t % p.n_tiles_n;
            const int e = p.tiles[2 * mt], row0 = p.tiles[2 * mt + 1];
            const int nrows = min(BM, p.offsets[e + 1] - row0);
            const int wrow0 = row0 + quad * 32;                      // this warp's 32 rows
            const int nvalid = max(0, min(32, nrows - quad * 32));
            float r0, r1;
            epi_prefetch<EPI>(p, e, nt, half, wrow0 + lane, lane < nvalid, sc, lane, r0, r1);
            if (!mbar_wait(&ctl->acc_full[buf], aph, abort, p.status, 4, t)) break;
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * BN);
            if (EPI == EPI_SWIGLU)
                epilogue_swiglu<FMT>(p, taddr, half, e, nt, wrow0, nvalid, stage, sc, r0, &ctl->acc_empty[buf],
                                     p.tma_c ? &tm_c : nullptr, lane);
            else
                epilogue_down<FMT>(p, taddr, half, e, nt, wrow0, nvalid, stage, sc, r0, r1, &ctl->acc_empty[buf],
                                   p.tma_c ? &tm_c : nullptr, lane);
            buf ^= 1;
            if (buf == 0) aph ^= 1;
        }
        if (lane == 0) tma_store_wait_all();     // this warp's bulk stores have landed
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// ------------------------------------------------------------------ CTA-pair grouped GEMM

// The same grouped GEMM on pairs of SMs: a cluster of two CTAs computes a
// 256-row x 256-column tile with one tcgen05.mma.cta_group::2 per K slice
// (M = 256: CTA r holds rows 128 r .. 128 r + 127 of A and columns
// 128 r .. 128 r + 127 of B in its shared memory, and its 128 rows of the
// accumulator in its tensor memory).  Each SM so loads half of the tile's
// weight columns and all of its own rows: 32 KB per 128-byte K block instead
// of 48 KB for the same MMA work, and six stages fit where four did.
// Tiles are the pair tiles of the routing metadata (256 rows of one expert;
// the second CTA's rows may be past the expert's last row, then they are
// computed and not stored).
//   warp 0 (both CTAs)   TMA producer for its own A rows and B columns; the
//                        loads signal the leader CTA's stage barrier, whose
//                        expected byte count covers both CTAs' loads
//   warp 1 (leader)      MMA issuer; each K block's commit is multicast to the
//                        stage-free barriers of both CTAs, each tile's to
//                        both CTAs' accumulator-full barriers
//   warps 2..9 (both)    epilogue on the CTA's own 128 rows; every warp
//                        releases the accumulator on the leader's barrier
//                        (16 arrivals per phase)
// Both CTAs allocate and free the tensor memory together (cta_group::2); a
// cluster barrier after set-up and before the free keeps either CTA from
// touching the other's barriers or memory while it does not exist.
constexpr int kStagesP = 6;
constexpr int kABytesP = BM * BK;             // 16 KB: this CTA's rows of A
constexpr int kBBytesP = (BN / 2) * BK;       // 16 KB: this CTA's half of the B columns
constexpr int kStageBytesP = kABytesP + kBBytesP;
constexpr size_t kSmemBytesP =
    (size_t)kStagesP * kStageBytesP + (size_t)kEpiWarps * kEpiStageBytes + 1024 + 256;

struct CtlP {
    uint64_t full[kStagesP];
    uint64_t empty[kStagesP];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// Instruction descriptor of the pair MMA: as idesc(), with M = 256.
template <int FMT>
__host__ __device__ constexpr uint32_t idesc_pair() {
    return (FMT == FMT_E4M3 ? (1u << 4) : ((2u << 4) | (1u << 7) | (1u << 10))) | ((uint32_t)(BN >> 3) << 17) |
           ((uint32_t)((2 * BM) >> 4) << 24);
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The address of this CTA's shared variable in the leader's (rank 0) shared memory.
__device__ __forceinline__ uint32_t leader_addr(const void* p) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(smem_u32(p)));
    return r;
}

// TMA load into this CTA's shared memory whose completion is counted on a
// barrier of the pair (here: the leader's stage barrier).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

template <int FMT>
__device__ __forceinline__ void mma_8bit_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accum) {
    if (FMT == FMT_E4M3)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
            "l"(adesc), "l"(bdesc), "r"(idesc_pair<FMT>()), "r"(accum));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
            "l"(adesc), "l"(bdesc), "r"(idesc_pair<FMT>()), "r"(accum));
}

// Arrive, when the pair MMAs issued so far are done, on `bar` in each CTA of
// `mask` (same shared-memory offset in each).
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar, uint16_t mask) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "h"(mask)
                 : "memory");
}

// try_wait with cluster-scope acquire: for barriers the other CTA arrives on.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort, int32_t* status, int site,
                                  int iter) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_timer();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort) return false;
        if (global_timer() - t0 > kWaitBudgetNs) {
            *abort = 1;
            report_timeout(status, site, iter, (int)parity);
            return false;
        }
    }
}

template <int EPI, int FMT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tc_pair_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_c, const TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    float* epi_stage = reinterpret_cast<float*>(smem + kStagesP * kStageBytesP);
    CtlP* ctl = reinterpret_cast<CtlP*>(smem + kStagesP * kStageBytesP + kEpiWarps * kEpiStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_ctarank();
    const bool leader = rank == 0;
    const int nkb = p.K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], 1);
            mbar_init(&ctl->acc_empty[b], 2 * kEpiWarps);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctl->tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    volatile int* abort = &ctl->abort;
    pdl_wait();
    pdl_trigger();
    const int num_tiles = p.meta[META_NPAIRS] * p.n_tiles_n;
    const int cid = (int)cluster_index(), ncl = (int)cluster_count();

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs): own rows of A, own half of B
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_par[kStagesP];
            bool issued[kStagesP];
            for (int i = 0; i < kStagesP; ++i) issued[i] = false;
            bool ok = true;
            for (int t = cid; t < num_tiles && ok; t += ncl) {
                const int mt = t / p.n_tiles_n, nt = t % p.n_tiles_n;
                const int e = p.pairs[2 * mt], row0 = p.pairs[2 * mt + 1] + rank * BM;
                const int brow = e * p.N + nt * BN + rank * (BN / 2);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&ctl->empty[s], ph ^ 1, abort, p.status, 1, t)) { ok = false; break; }
                    if (leader) mbar_arrive_expect_tx(&ctl->full[s], 2 * kStageBytesP);
                    const uint32_t bar = leader_addr(&ctl->full[s]);
                    uint8_t* sa = smem + s * kStageBytesP;
                    tma_load_2d_pair(sa, &tm_a, bar, kb * BK, row0);
                    tma_load_2d_pair(sa + kABytesP, &tm_b, bar, 0, tiled_row(brow, kb, nkb));
                    issued[s] = true;
                    issued_par[s] = ph;
                    if (++s == kStagesP) { s = 0; ph ^= 1; }
                }
            }
            if (leader) {
                // the leader's stage barriers count both CTAs' bytes: wait for the
                // copies of every stage it issued to land (bounded)
                for (int i = 0; i < kStagesP; ++i) {
                    if (!issued[i]) continue;
                    const uint64_t t0 = global_timer();
                    while (!mbar_try_wait(&ctl->full[i], issued_par[i]) && global_timer() - t0 < kWaitBudgetNs) {}
                }
            }
            if (!ok) {
                // after a timeout, copies this CTA issued may still be in flight and
                // their completion is counted only on the other CTA's barrier: give
                // them time to land before the CTA can exit (bounded)
                const uint64_t t0 = global_timer();
                while (global_timer() - t0 < 200000ull) {}
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------- MMA issuer (leader CTA only)
            int s = 0, buf = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true;
            for (int t = cid; t < num_tiles && ok; t += ncl) {
                if (!mbar_wait_cluster(&ctl->acc_empty[buf], aph ^ 1, abort, p.status, 2, t)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(buf * BN);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&ctl->full[s], ph, abort, p.status, 3, t)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * kStageBytesP);
                    const uint32_t b_addr = a_addr + kABytesP;
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)
                        mma_8bit_pair<FMT>(d_tmem, desc_sw128(a_addr + kk * 32), desc_sw128(b_addr + kk * 32),
                                           (kb | kk) != 0 ? 1u : 0u);
                    mma_commit_pair(&ctl->empty[s], 0x3);
                    if (++s == kStagesP) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                mma_commit_pair(&ctl->acc_full[buf], 0x3);
                buf ^= 1;
                if (buf == 0) aph ^= 1;
            }
            // all MMAs issued by this thread complete before the tensor memory is freed (bounded)
            mma_commit_pair(&ctl->drain, 0x1);
            const uint64_t t0 = global_timer();
            while (!mbar_try_wait(&ctl->drain, 0) && global_timer() - t0 < kWaitBudgetNs) {}
        }
    } else {
        // ---------------- epilogue warps (both CTAs): this CTA's 128 rows of the tile
        const int ew = warp - 2;
        const int quad = warp & 3;
        const int half = ew >> 2;
        float* stage = epi_stage + ew * (kEpiStageBytes / 4);
        int buf = 0;
        uint32_t aph = 0;
        float* sc = stage + kEpiStoreBytes / 4;
        for (int t = cid; t < num_tiles; t += ncl) {
            const int mt = t / p.n_tiles_n, nt = t % p.n_tiles_n;
            const int e = p.pairs[2 * mt], row0 = p.pairs[2 * mt + 1] + rank * BM;
            const int nrows = min(BM, p.offsets[e + 1] - row0);
            const int wrow0 = row0 + quad * 32;
            const int nvalid = max(0, min(32, nrows - quad * 32));
            float r0, r1;
            epi_prefetch<EPI>(p, e, nt, half, wrow0 + lane, lane < nvalid, sc, lane, r0, r1);
            if (!mbar_wait(&ctl->acc_full[buf], aph, abort, p.status, 4, t)) break;
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * BN);
            if (EPI == EPI_SWIGLU)
                epilogue_swiglu<FMT, true>(p, taddr, half, e, nt, wrow0, nvalid, stage, sc, r0,
                                           &ctl->acc_empty[buf], p.tma_c ? &tm_c : nullptr, lane);
            else
                epilogue_down<FMT, true>(p, taddr, half, e, nt, wrow0, nvalid, stage, sc, r0, r1,
                                         &ctl->acc_empty[buf], p.tma_c ? &tm_c : nullptr, lane);
            buf ^= 1;
            if (buf == 0) aph ^= 1;
        }
        if (lane == 0) tma_store_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// ------------------------------------------------------------------ fused expert FFN (few rows)

// Requantise the rows [row0, row0 + nrows) of h with one warp: the same
// arithmetic as requant_kernel (sh = max of the row's npart partial maxima /
// qmax, codes of h / sh).  Reads through L2 (other CTAs wrote h and the maxima).
// Lane r finds the scale of rows r, r + 32, ... (kept in `scales`, nrows <=
// 128); then one flat pass over the rows' h with 8 x 16-byte loads per lane
// in flight, so a few rows cost a few L2 round trips in total.
template <int FMT>
__device__ void requant_rows_warp(const float* h32, const float* pamax, int f, int npart, int row0, int nrows,
                                  int8_t* hq, float* sh, float* scales, int lane) {
    constexpr int kB = 8;
    const int n4 = f / 4;
    for (int r = lane; r < nrows; r += 32) {
        const float* pm = pamax + (int64_t)(row0 + r) * npart;
        float m = 0.0f;
        for (int i = 0; i < npart; ++i) m = fmaxf(m, __ldcg(pm + i));
        const float s = m > 0.0f ? __fdiv_rn(m, fmt_qmax<FMT>()) : 0.0f;
        scales[r] = s;
        sh[row0 + r] = s;
    }
    __syncwarp();
    const int total = nrows * n4;   // float4 groups of all rows
    const float4* h4 = reinterpret_cast<const float4*>(h32 + (int64_t)row0 * f);
    uint32_t* q4 = reinterpret_cast<uint32_t*>(hq + (int64_t)row0 * f);
    for (int b = 0; b < total; b += 32 * kB) {
        float4 h[kB];
#pragma unroll
        for (int i = 0; i < kB; ++i)
            if (b + lane + 32 * i < total) h[i] = __ldcg(h4 + b + lane + 32 * i);
#pragma unroll
        for (int i = 0; i < kB; ++i) {
            const int j = b + lane + 32 * i;
            if (j < total) {
                const float s = scales[j / n4];
                const float rs = s > 0.0f ? __frcp_rn(s) : 0.0f;
                q4[j] = s > 0.0f ? fmt_codes4<FMT>(h[i].x, h[i].y, h[i].z, h[i].w, s, rs) : 0u;
            }
        }
    }
}

// A release add whose old value nobody waits for.
__device__ __forceinline__ void red_release_add(int32_t* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int32_t* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int32_t* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Orders this thread's generic-proxy global accesses with its async-proxy
// (TMA) ones: after h codes are stored (before they are released), and after
// they are acquired (before a TMA load reads them).
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

struct FusedExtra {
    int32_t* count;   // [m-tiles] GEMM1 epilogue-warp arrivals
    int32_t* ready;   // [m-tiles] 1 once the m-tile's h codes are written
    int32_t* qhead;   // next m-tile a requantisation warp takes
    int32_t* next;    // next tile to take (dynamic schedule)
    int8_t* hq;       // [rows][f] h codes
    float* sh;        // [rows] h scales
    uint64_t budget_ns;   // bound on each wait for another block's results (counts, ready flags)
    int skip_ready;       // testing aid: the m-tile whose ready flag is never released (-1: none)
};                    // (count, ready, qhead, next zeroed before the launch)

constexpr int kFusedThreads = kThreads + 32;   // + one requantisation warp (warp 10)
constexpr int kTileRing = 8;                   // tiles taken but not yet finished, per CTA

// The order in which a CTA's producer took its tiles, for its MMA and epilogue warps.
struct TileRing {
    uint64_t full[kTileRing];    // the producer wrote tile[q]
    uint64_t empty[kTileRing];   // the MMA thread and the 8 epilogue warps have read it
    int tile[kTileRing];         // tile index, or -1 = no more tiles
};
// Shared-memory plan of the fused launch: per stage the tile's token rows
// (128, or 32 in the swapped-operand plan) then its 256 weight rows, each
// 128 bytes of K.
template <bool SW>
struct FusedPlan {
    static constexpr int kT = (SW ? kFusedSwapRows : BM) * BK;
    static constexpr int kStage = kT + kBBytes;
    static constexpr int kNStages = kStages;
    static constexpr size_t kSmem =
        (size_t)kNStages * kStage + (size_t)(kEpiWarps + 1) * kEpiStageBytes + 1024 + 256 + 256;
    static_assert(kSmem <= 232448, "shared memory per block");
    static_assert(kT % 1024 == 0 && kStage % 1024 == 0, "128-byte swizzle atoms stay aligned");
};

// GEMM1 (gate/up + SwiGLU), the row-wise requantisation of h and GEMM2 (down)
// in one persistent launch, for launches with few rows per expert (decode),
// where both GEMMs stream weights and a separate GEMM2 launch would wait for
// the partial last wave of GEMM1 to drain.  One tile index space: GEMM1 tiles
// (m-tile x 256 gate/up columns) first, then GEMM2 tiles (m-tile x 256 output
// columns), dealt round robin, so the SMs idle in GEMM1's last wave start on
// GEMM2 tiles at once.  Tiles are taken from a device-wide counter in that
// order (each CTA's producer takes the next one when it has room and hands the
// index to its MMA and epilogue warps through a small ring), so every tile a
// wait depends on has already been taken by a running CTA: the launch makes
// progress even when not all its CTAs are resident.  Dependencies are per
// m-tile (one expert's rows): every
// epilogue warp that finishes a GEMM1 tile adds one to count[m] (a release add
// whose result it does not wait for).  Warp 10 of every CTA takes m-tiles in
// index order from a counter, waits until the m-tile's count is complete
// (GEMM1 column tiles x epilogue warps), requantises its rows and releases
// ready[m], so requantisation runs on otherwise idle warps of many CTAs and
// never delays an epilogue (when the epilogue warp that completed an m-tile
// requantised it itself, it fell behind, became the last arrival again, and
// the delays piled up; when the last arrival found out by an atomic's result
// and queued the m-tile, every epilogue warp waited for that result).  The producer of a GEMM2 tile waits
// for ready[m] (bounded by the handle's wait budget) before loading its h codes.  GEMM1 tiles are all taken
// before any GEMM2 tile, GEMM1 tiles wait on nothing, and the requant warps
// wait only on GEMM1 tiles, so the waits always end.  Arithmetic per element
// is that of the two separate kernels and requant_kernel, so the results are
// identical.
template <int FMT, bool SW>
__global__ void __launch_bounds__(kFusedThreads, 1)
    tc_ffn_fused_kernel(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_b1,
                        const __grid_constant__ CUtensorMap tm_a2, const __grid_constant__ CUtensorMap tm_b2,
                        const TcParams p1, const TcParams p2, const FusedExtra fx) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    using Plan = FusedPlan<SW>;
    constexpr int NS = Plan::kNStages;
    float* epi_stage = reinterpret_cast<float*>(smem + NS * Plan::kStage);
    // the requantisation warp's scale buffer follows the epilogue warps' staging buffers
    CtlT<NS>* ctl = reinterpret_cast<CtlT<NS>*>(smem + NS * Plan::kStage + (kEpiWarps + 1) * kEpiStageBytes);
    TileRing* ring = reinterpret_cast<TileRing*>(reinterpret_cast<uint8_t*>(ctl) + 256);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], 1);
            mbar_init(&ctl->acc_empty[b], kEpiWarps);
        }
        for (int q = 0; q < kTileRing; ++q) {
            mbar_init(&ring->full[q], 1);
            mbar_init(&ring->empty[q], 1 + kEpiWarps);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctl->tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    volatile int* abort = &ctl->abort;
    pdl_wait();
    pdl_trigger();
    const int n_mt = p1.meta[META_NTILES];
    const int w1 = n_mt * p1.n_tiles_n;
    const int num_tiles = w1 + n_mt * p2.n_tiles_n;
    const int arrivals = p1.n_tiles_n * kEpiWarps;   // per m-tile, when its h is complete

    // tile t -> (first GEMM?, m-tile, column tile)
    auto decode = [&](int t, bool& g1, int& mt, int& nt) {
        g1 = t < w1;
        const int u = g1 ? t : t - w1;
        const int nn = g1 ? p1.n_tiles_n : p2.n_tiles_n;
        mt = u / nn;
        nt = u % nn;
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_par[NS];
            bool issued[NS];
            for (int i = 0; i < NS; ++i) issued[i] = false;
            bool ok = true;
            int q = 0;
            uint32_t rph = 0;
            while (ok) {
                // take the next tile and tell the MMA and epilogue warps
                int t = atomicAdd(fx.next, 1);
                if (t >= num_tiles) t = -1;
                if (!mbar_wait(&ring->empty[q], rph ^ 1, abort, p1.status, 8, t)) break;
                ring->tile[q] = t;
                mbar_arrive(&ring->full[q]);
                if (++q == kTileRing) { q = 0; rph ^= 1; }
                if (t < 0) break;
                bool g1;
                int mt, nt;
                decode(t, g1, mt, nt);
                const TcParams& p = g1 ? p1 : p2;
                const CUtensorMap* ma = g1 ? &tm_a1 : &tm_a2;
                const CUtensorMap* mb = g1 ? &tm_b1 : &tm_b2;
                const int e = p.tiles[2 * mt], row0 = p.tiles[2 * mt + 1];
                const int brow = e * p.N + nt * BN;
                if (!g1) {
                    // this m-tile's h codes must be written before they are loaded
                    const uint64_t t0 = global_timer();
                    while (ld_acquire(fx.ready + mt) == 0) {
                        if (*abort) { ok = false; break; }
                        if (global_timer() - t0 > fx.budget_ns) {
                            *abort = 1;
                            report_timeout(p.status, 6, t, mt);
                            ok = false;
                            break;
                        }
                    }
                    if (!ok) break;
                    fence_proxy_async_global();
                }
                if (SW && p.offsets[e + 1] - row0 > kFusedSwapRows) {
                    // more rows than the swapped plan's token tile holds (the host's
                    // choice of plan excludes it): report and stop
                    atomicExch(p.status, (int32_t)MOE_ERR_INVALID_ARG);
                    if (atomicCAS(p.status + 1, 0, 17) == 0) {
                        p.status[2] = (int32_t)blockIdx.x;
                        p.status[3] = mt;
                        p.status[4] = p.offsets[e + 1] - row0;
                    }
                    *abort = 1;
                    break;
                }
                const int nkb = p.K / BK;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&ctl->empty[s], ph ^ 1, abort, p.status, 1, t)) { ok = false; break; }
                    mbar_arrive_expect_tx(&ctl->full[s], Plan::kStage);
                    uint8_t* sa = smem + s * Plan::kStage;
                    tma_load_2d(sa, ma, &ctl->full[s], kb * BK, row0);
                    tma_load_2d(sa + Plan::kT, mb, &ctl->full[s], kb * BK, brow);
                    issued[s] = true;
                    issued_par[s] = ph;
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
            }
            for (int i = 0; i < NS; ++i) {
                if (!issued[i]) continue;
                const uint64_t t0 = global_timer();
                while (!mbar_try_wait(&ctl->full[i], issued_par[i]) && global_timer() - t0 < kWaitBudgetNs) {}
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            int s = 0, buf = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true;
            int q = 0;
            uint32_t rph = 0;
            while (ok) {
                if (!mbar_wait(&ring->full[q], rph, abort, p1.status, 9, 0)) break;
                const int t = ring->tile[q];
                mbar_arrive(&ring->empty[q]);
                if (++q == kTileRing) { q = 0; rph ^= 1; }
                if (t < 0) break;
                const int nkb = (t < w1 ? p1.K : p2.K) / BK;
                if (!mbar_wait(&ctl->acc_empty[buf], aph ^ 1, abort, p1.status, 2, t)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(buf * (SW ? 2 * kFusedSwapRows : BN));
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&ctl->full[s], ph, abort, p1.status, 3, t)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t t_addr = smem_u32(smem + s * Plan::kStage);
                    const uint32_t w_addr = t_addr + Plan::kT;
                    if (SW) {
                        // weights as A (two 128-row halves), token rows as B (N = 32)
                        constexpr uint32_t id = idesc<FMT, BM, kFusedSwapRows>();
#pragma unroll
                        for (int kk = 0; kk < BK / 32; ++kk) {
                            const uint64_t bd = desc_sw128(t_addr + kk * 32);
                            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
                            mma_8bit<FMT, id>(d_tmem, desc_sw128(w_addr + kk * 32), bd, acc);
                            mma_8bit<FMT, id>(d_tmem + kFusedSwapRows, desc_sw128(w_addr + BM * BK + kk * 32), bd,
                                              acc);
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < BK / 32; ++kk)
                            mma_8bit<FMT>(d_tmem, desc_sw128(t_addr + kk * 32), desc_sw128(w_addr + kk * 32),
                                          (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(&ctl->empty[s]);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                mma_commit(&ctl->acc_full[buf]);
                buf ^= 1;
                if (buf == 0) aph ^= 1;
            }
            mma_commit(&ctl->drain);
            const uint64_t t0 = global_timer();
            while (!mbar_try_wait(&ctl->drain, 0) && global_timer() - t0 < kWaitBudgetNs) {}
        }
    } else if (warp == kFusedThreads / 32 - 1) {
        // ---------------- requantisation warp: m-tiles in index order
        float* scales = epi_stage + kEpiWarps * (kEpiStageBytes / 4);
        while (true) {
            int i = 0;
            if (lane == 0) i = atomicAdd(fx.qhead, 1);
            i = __shfl_sync(0xffffffffu, i, 0);
            if (i >= n_mt) break;
            int ok = 1;
            if (lane == 0) {
                const uint64_t t0 = global_timer();
                while (ld_acquire(fx.count + i) < arrivals) {
                    if (*abort) { ok = 0; break; }
                    if (global_timer() - t0 > fx.budget_ns) {
                        *abort = 1;
                        report_timeout(p1.status, 7, i, 0);
                        ok = 0;
                        break;
                    }
                    __nanosleep(64);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            (void)ld_acquire(fx.count + i);   // each lane's own acquire of the m-tile's h
            const int mt = i;
            const int e = p1.tiles[2 * mt], row0 = p1.tiles[2 * mt + 1];
            const int nrows = min(BM, p1.offsets[e + 1] - row0);
            requant_rows_warp<FMT>(p1.h32, p1.pamax, p1.f, p1.f / (SW ? 32 : 64), row0, nrows, fx.hq, fx.sh, scales,
                                   lane);
            // the codes reach the GEMM2 producers' TMA loads (async proxy) and the
            // epilogues' loads through lane 0's release after the warp barrier
            fence_proxy_async_global();
            __syncwarp();
            if (lane == 0 && mt != fx.skip_ready) st_release(fx.ready + mt, 1);
        }
    } else {
        // ---------------- epilogue warps
        const int ew = warp - 2;
        const int quad = warp & 3;
        const int half = ew >> 2;
        float* stage = epi_stage + ew * (kEpiStageBytes / 4);
        float* sc = stage + kEpiStoreBytes / 4;
        int buf = 0;
        uint32_t aph = 0;
        int q = 0;
        uint32_t rph = 0;
        while (true) {
            if (!mbar_wait(&ring->full[q], rph, abort, p1.status, 10, 0)) break;
            const int t = ring->tile[q];
            __syncwarp();
            if (lane == 0) mbar_arrive(&ring->empty[q]);
            if (++q == kTileRing) { q = 0; rph ^= 1; }
            if (t < 0) break;
            bool g1;
            int mt, nt;
            decode(t, g1, mt, nt);
            const TcParams& p = g1 ? p1 : p2;
            const int e = p.tiles[2 * mt], row0 = p.tiles[2 * mt + 1];
            const int nrows = min(BM, p.offsets[e + 1] - row0);
            const int wrow0 = row0 + quad * 32;
            const int nvalid = max(0, min(32, nrows - quad * 32));
            float r0, r1, c0 = 0.0f, c1 = 0.0f;
            if (g1) {
                if (SW) {
                    // the lane's gate / up channel scales; lane j < 16: row 16 half + j's activation scale
                    const int ch = nt * 128 + 32 * quad + lane;
                    c0 = p1.sw0[(int64_t)e * p1.f + ch];
                    c1 = p1.sw1[(int64_t)e * p1.f + ch];
                    const int r = 16 * half + lane;
                    r0 = lane < 16 && r < nrows ? p1.sx[p1.row2ts[row0 + r] / p1.k] : 0.0f;
                    r1 = 0.0f;
                } else {
                    epi_prefetch<EPI_SWIGLU>(p1, e, nt, half, wrow0 + lane, lane < nvalid, sc, lane, r0, r1);
                }
            } else {
                // the h scales this epilogue reads are released with the m-tile's ready flag:
                // wait for it (bounded) before fetching them
                int rdy = 0;
                if (lane == 0) {
                    const uint64_t t0 = global_timer();
                    while ((rdy = ld_acquire(fx.ready + mt)) == 0) {
                        if (*abort) break;
                        if (global_timer() - t0 > fx.budget_ns) {
                            *abort = 1;
                            report_timeout(p2.status, 16, t, mt);
                            break;
                        }
                    }
                }
                rdy = __shfl_sync(0xffffffffu, rdy, 0);
                if (rdy == 0) break;
                (void)ld_acquire(fx.ready + mt);   // each lane's own acquire of the released scales
                if (SW) {
                    // the lane's output column scale; lane r: row r's h scale and routing weight
                    c0 = p2.sw0[(int64_t)e * p2.N + nt * BN + 128 * half + 32 * quad + lane];
                    r0 = lane < nrows ? p2.sh[row0 + lane] : 0.0f;
                    r1 = lane < nrows ? p2.topk_w[p2.row2ts[row0 + lane]] : 0.0f;
                } else {
                    epi_prefetch<EPI_DOWN>(p2, e, nt, half, wrow0 + lane, lane < nvalid, sc, lane, r0, r1);
                }
            }
            if (!mbar_wait(&ctl->acc_full[buf], aph, abort, p1.status, 4, t)) break;
            tc_fence_after();
            const uint32_t taddr =
                tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * (SW ? 2 * kFusedSwapRows : BN));
            if (g1) {
                if (SW)
                    epilogue_swiglu_sw<FMT>(p1, taddr, half, quad, nt, row0, nrows, c0, c1, r0, &ctl->acc_empty[buf],
                                            lane);
                else
                    epilogue_swiglu<FMT>(p1, taddr, half, e, nt, wrow0, nvalid, stage, sc, r0, &ctl->acc_empty[buf],
                                         nullptr, lane);
                // this warp's share of the tile is stored: count it.  The lanes' stores are
                // ordered before lane 0's release by the warp barrier (it orders the
                // participating lanes' memory accesses), and a release publishes everything
                // ordered before it, so no separate fence is needed (membar.gl here cost the
                // decode step about 5 us with the requantisation warp's below)
                __syncwarp();
                if (lane == 0) red_release_add(fx.count + mt, 1);
            } else if (SW) {
                epilogue_down_sw<FMT>(p2, taddr, half, quad, nt, row0, nrows, c0, r0, r1, &ctl->acc_empty[buf], lane);
            } else {
                epilogue_down<FMT>(p2, taddr, half, e, nt, wrow0, nvalid, stage, sc, r0, r1, &ctl->acc_empty[buf],
                                   nullptr, lane);
            }
            buf ^= 1;
            if (buf == 0) aph ^= 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// ------------------------------------------------------------------ requantisation of h

// One warp per sorted row: sh = max over the row's partial maxima / 127 and
// codes rint(h / sh), ties to even, clamped to +-127 (sh = 0 gives 0).  The
// scale comes from the partial maxima, not from h, so a row's h loads (up to
// kRqBatch x 16 bytes per lane) and its partial-maximum loads are issued
// together; further batches follow (f = 1536: 12 x 16 bytes per lane in three
// batches; 4 per batch measured faster than 6, 8 or 12: 39 registers, so 6
// blocks of 8 warps per SM).  A small batch keeps the registers, and so the warps per SM that
// hide the per-element arithmetic, in balance with the bytes in flight.
constexpr int kRqThreads = 256;
constexpr int kRqBatch = 4;

template <int FMT>
__global__ void __launch_bounds__(kRqThreads) requant_kernel(const float* __restrict__ h32,
                                                             const float* __restrict__ pamax, int f,
                                                             const int32_t* __restrict__ meta,
                                                             int8_t* __restrict__ hq,
                                                             float* __restrict__ sh) {
    pdl_wait();
    pdl_trigger();

    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (kRqThreads / 32) + (threadIdx.x >> 5);
    if (row >= meta[META_R]) return;
    const int npart = f / 64, n4 = f / 4;
    const float4* hrow = reinterpret_cast<const float4*>(h32 + (int64_t)row * f);
    uint32_t* qrow = reinterpret_cast<uint32_t*>(hq + (int64_t)row * f);
    float4 h[kRqBatch];
#pragma unroll
    for (int i = 0; i < kRqBatch; ++i) {
        const int c4 = lane + 32 * i;
        if (c4 < n4) h[i] = hrow[c4];
    }
    float m = 0.0f;
    for (int i = lane; i < npart; i += 32) m = fmaxf(m, pamax[(int64_t)row * npart + i]);
    m = warp_max(m);
    const float s = m > 0.0f ? __fdiv_rn(m, fmt_qmax<FMT>()) : 0.0f;
    const float rs = s > 0.0f ? __frcp_rn(s) : 0.0f;
    if (lane == 0) sh[row] = s;
    for (int b = 0; b < n4; b += 32 * kRqBatch) {
        if (b > 0) {
#pragma unroll
            for (int i = 0; i < kRqBatch; ++i) {
                const int c4 = b + lane + 32 * i;
                if (c4 < n4) h[i] = hrow[c4];
            }
        }
#pragma unroll
        for (int i = 0; i < kRqBatch; ++i) {
            const int c4 = b + lane + 32 * i;
            if (c4 < n4)
                qrow[c4] = s > 0.0f ? fmt_codes4<FMT>(h[i].x, h[i].y, h[i].z, h[i].w, s, rs) : 0u;
        }
    }
}

// ------------------------------------------------------------------ approximate router logits

// Approximate router logits on the tensor cores, for the certified router:
// l~[t][e] = sum_j x[t][j] (hi[e][j] + lo[e][j]) with W_g split into two bf16
// parts (hi = bf16(w), lo = bf16(w - hi), so |w - hi - lo| <= 2^-16 |w|),
// tcgen05.mma kind::f16 (bf16 x bf16, fp32 accumulators in TMEM).  One CTA per
// 128 tokens and 64 experts (a 256-expert router is four CTAs per token block,
// so wide routers still fill the GPU): warp 0 loads X (128 x 64 bf16) and both
// W parts (EPAD x 64 bf16) per k-block by TMA into a ring, warp 1 issues two
// MMAs per 16 channels into one accumulator, warps 2-5 write the EPAD columns
// of their 32 rows.  These
// values only choose candidates; the logits that decide top-k and the gate
// weights are recomputed in the stated fp32 order (router_select_kernel).
constexpr int kRcBK = 64;                     // bf16 channels per k-block (128 bytes)
constexpr int kRcThreads = 192;
constexpr int kRcABytes = BM * kRcBK * 2;     // 16 KB
constexpr int kRcSlice = 64;                  // experts per CTA (the padded router is a multiple)

template <int EPAD>
struct RcCfg {
    static constexpr int kBBytes = EPAD * kRcBK * 2;                  // one W part
    static constexpr int kStage = kRcABytes + 2 * kBBytes;
    static constexpr int kStages = EPAD <= 64 ? 4 : (EPAD <= 128 ? 3 : 2);
    static constexpr size_t kSmem = (size_t)kStages * kStage + 1024 + 256;
    // kind::f16: D = f32 (bits 4-5 = 1), A and B bf16 (bits 7-9, 10-12 = 1), K-major
    static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(EPAD >> 3) << 17) |
                                       ((uint32_t)(BM >> 4) << 24);
};

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum));
}

template <int EPAD>
__global__ void __launch_bounds__(kRcThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_hi,
                     const __grid_constant__ CUtensorMap tm_lo, int T, int d, int E, float* __restrict__ approx,
                     int32_t* status) {
    using C = RcCfg<EPAD>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + C::kStages * C::kStage);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // blockIdx.x: which EPAD experts (a slice of the padded router), blockIdx.y:
    // which 128 tokens; the slices of one token block are neighbours in launch
    // order, so they read the block's X from L2
    const int e0 = blockIdx.x * EPAD;
    const int t0 = blockIdx.y * BM;
    const int nkb = d / kRcBK;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        mbar_init(&ctl->acc_full[0], 1);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctl->tmem_base)),
                     "r"((uint32_t)EPAD));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    volatile int* abort = &ctl->abort;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_par[4];
            bool issued[4] = {false, false, false, false};
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(&ctl->empty[s], ph ^ 1, abort, status, 11, kb)) break;
                mbar_arrive_expect_tx(&ctl->full[s], C::kStage);
                uint8_t* sa = smem + s * C::kStage;
                tma_load_2d(sa, &tm_x, &ctl->full[s], kb * kRcBK, t0);
                tma_load_2d(sa + kRcABytes, &tm_hi, &ctl->full[s], kb * kRcBK, e0);
                tma_load_2d(sa + kRcABytes + C::kBBytes, &tm_lo, &ctl->full[s], kb * kRcBK, e0);
                issued[s] = true;
                issued_par[s] = ph;
                if (++s == C::kStages) { s = 0; ph ^= 1; }
            }
            for (int i = 0; i < C::kStages; ++i) {
                if (!issued[i]) continue;
                const uint64_t tw = global_timer();
                while (!mbar_try_wait(&ctl->full[i], issued_par[i]) && global_timer() - tw < kWaitBudgetNs) {}
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(&ctl->full[s], ph, abort, status, 12, kb)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + s * C::kStage);
                const uint32_t hi_addr = a_addr + kRcABytes, lo_addr = hi_addr + C::kBBytes;
#pragma unroll
                for (int kk = 0; kk < kRcBK / 16; ++kk) {
                    mma_bf16(tmem, desc_sw128(a_addr + kk * 32), desc_sw128(hi_addr + kk * 32), C::kIdesc,
                             (kb | kk) != 0 ? 1u : 0u);
                    mma_bf16(tmem, desc_sw128(a_addr + kk * 32), desc_sw128(lo_addr + kk * 32), C::kIdesc, 1u);
                }
                mma_commit(&ctl->empty[s]);
                if (++s == C::kStages) { s = 0; ph ^= 1; }
            }
            if (ok) mma_commit(&ctl->acc_full[0]);
            mma_commit(&ctl->drain);
            const uint64_t tw = global_timer();
            while (!mbar_try_wait(&ctl->drain, 0) && global_timer() - tw < kWaitBudgetNs) {}
        }
    } else {
        // warps 2..5: TMEM lane quarter warp % 4 = 32 tokens each
        const int quad = warp & 3;
        if (mbar_wait(&ctl->acc_full[0], 0, abort, status, 13, 0)) {
            tc_fence_after();
            const int t = t0 + quad * 32 + lane;
#pragma unroll 1
            for (int c0 = 0; c0 < EPAD; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)c0, v);
                tmem_ld_wait();
                if (t < T)
                    for (int j = 0; j < 32; ++j)
                        if (e0 + c0 + j < E) approx[(int64_t)t * E + e0 + c0 + j] = __uint_as_float(v[j]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)EPAD));
    }
}

// ------------------------------------------------------------------ tensor-core rate

// The dense 8-bit tensor-core rate of this GPU as this library's own MMAs
// reach it: one CTA per SM; the A (128 x 128 B) and B (256 x 128 B) tiles of
// one k-block of the grouped GEMMs, filled once with pseudo-random codes (the
// switching activity, hence the power draw and the clock, of real operands),
// stay in shared memory; one thread issues n_mma M=128 x N=256 x K=32 MMAs
// back to back, stepping through the k-block's four K slices as the GEMMs do,
// into one 256-column TMEM accumulator (restarted every 1024 MMAs so the
// sums stay bounded).  No copies, no epilogue: the loop is the tensor pipe
// alone.  The final commit is waited for (bounded) before TMEM is freed.
constexpr int kPeakThreads = 128;
constexpr size_t kPeakSmem = (size_t)kABytes + kBBytes + 1024 + 256;
constexpr uint64_t kPeakDrainNs = 10000000000ull;   // 10 s

template <int FMT>
__global__ void __launch_bounds__(kPeakThreads, 1) tc_peak_kernel(int64_t n_mma) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + kABytes + kBBytes);
    const int warp = threadIdx.x >> 5;
    // pseudo-random codes; E4M3 codes keep exponent field < 15 (finite, no NaN)
    uint32_t* w32 = reinterpret_cast<uint32_t*>(smem);
    for (int i = threadIdx.x; i < (kABytes + kBBytes) / 4; i += blockDim.x) {
        uint32_t h = (uint32_t)i * 0x9E3779B1u + blockIdx.x * 0x85EBCA77u;
        h ^= h >> 15;
        h *= 0x2C1B3C6Du;
        h ^= h >> 13;
        w32[i] = FMT == FMT_E4M3 ? (h & 0xB7B7B7B7u) : h;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (threadIdx.x == 0) {
        mbar_init(&ctl->drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctl->tmem_base)),
                     "r"((uint32_t)BN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    if (threadIdx.x == 0) {
        const uint32_t a_addr = smem_u32(smem), b_addr = a_addr + kABytes;
        for (int64_t i = 0; i < n_mma; ++i) {
            const int kk = (int)(i & 3);
            mma_8bit<FMT>(tmem, desc_sw128(a_addr + kk * 32), desc_sw128(b_addr + kk * 32), (i & 1023) ? 1u : 0u);
        }
        mma_commit(&ctl->drain);
        const uint64_t t0 = global_timer();
        while (!mbar_try_wait(&ctl->drain, 0) && global_timer() - t0 < kPeakDrainNs) {}
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)BN));
    }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D map over an int8 [rows][K] K-major matrix, box = box_rows x 128 bytes,
// 128-byte swizzle (the layout the MMA descriptors expect).
bool make_map(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {K, rows};
    const cuuint64_t strides[1] = {K};
    const cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a bf16 [rows][K] K-major matrix, box = box_rows x 64 elements
// (128 bytes), 128-byte swizzle.
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {K, rows};
    const cuuint64_t strides[1] = {K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kRcBK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a row-major [rows][cols] fp32 or bf16 output whose box is 32
// rows x 64 bytes (16 fp32 or 32 bf16 values) with 64-byte swizzle: the
// layout the epilogue warps stage a chunk of their 32 rows in.
bool make_out_map(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows, bool bf16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const uint64_t esz = bf16 ? 2 : 4;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * esz};
    const cuuint32_t box[2] = {(cuuint32_t)(64 / esz), 32};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPAD>
cudaError_t launch_router_tc_pad(const CUtensorMap& mx, const moe_w8a8_weights* w, int T, float* approx,
                                 cudaStream_t s) {
    using C = RcCfg<EPAD>;
    static std::atomic<uint64_t> attr{0};
    cudaError_t e = smem_attr_once(router_tc_kernel<EPAD>, C::kSmem, attr);
    if (e != cudaSuccess) return e;
    return launch_pdl(router_tc_kernel<EPAD>, dim3(w->rt_epad / EPAD, (T + BM - 1) / BM), dim3(kRcThreads), C::kSmem,
                      s, mx,
                      w->tm_rt_hi, w->tm_rt_lo, T, w->cfg.d, w->cfg.n_experts, approx, w->status);
}

template <int EPI, int FMT>
cudaError_t launch_fmt(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const TcParams& p,
                       int grid, cudaStream_t s) {
    static std::atomic<uint64_t> attr{0};
    cudaError_t e = smem_attr_once(tc_gemm_kernel<EPI, FMT>, kSmemBytes, attr);
    if (e != cudaSuccess) return e;
    return launch_pdl(tc_gemm_kernel<EPI, FMT>, dim3(grid), dim3(kThreads), kSmemBytes, s, ta, tb, tc, p);
}

template <int EPI>
cudaError_t launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const TcParams& p,
                   int grid, int fmt, cudaStream_t s) {
    return fmt == FMT_E4M3 ? launch_fmt<EPI, FMT_E4M3>(ta, tb, tc, p, grid, s)
                           : launch_fmt<EPI, FMT_INT8>(ta, tb, tc, p, grid, s);
}

// The pair kernel on as many SM pairs as can be resident at once (one pair
// per cluster of two CTAs; persistent), at most one per pair tile x column tile.
template <int EPI, int FMT>
cudaError_t launch_pair_fmt(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const TcParams& p,
                            int max_units, cudaStream_t s) {
    static std::atomic<uint64_t> attr{0};
    static int clusters[64] = {};
    auto kern = tc_pair_gemm_kernel<EPI, FMT>;
    cudaError_t e = smem_attr_once(kern, kSmemBytesP, attr);
    if (e != cudaSuccess) return e;
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int& nc = clusters[dev & 63];
    if (nc == 0) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(2);
        q.blockDim = dim3(kThreads);
        q.dynamicSmemBytes = kSmemBytesP;
        cudaLaunchAttribute a[1];
        a[0].id = cudaLaunchAttributeClusterDimension;
        a[0].val.clusterDim.x = 2;
        a[0].val.clusterDim.y = 1;
        a[0].val.clusterDim.z = 1;
        q.attrs = a;
        q.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, (const void*)kern, &q);
        if (e != cudaSuccess) return e;
        if (n <= 0) return cudaErrorInvalidConfiguration;
        nc = n;
    }
    const int grid = 2 * std::max(1, std::min(nc, max_units));
    return launch_pdl(kern, dim3(grid), dim3(kThreads), kSmemBytesP, s, ta, tb, tc, p);
}

template <int EPI>
cudaError_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const TcParams& p,
                        int max_units, int fmt, cudaStream_t s) {
    return fmt == FMT_E4M3 ? launch_pair_fmt<EPI, FMT_E4M3>(ta, tb, tc, p, max_units, s)
                           : launch_pair_fmt<EPI, FMT_INT8>(ta, tb, tc, p, max_units, s);
}

}  // namespace

bool tc_make_weight_maps(moe_w8a8_weights* w) {
    const moe_w8a8_config& c = w->cfg;
    const uint64_t E = w->n_local, d = c.d, f = c.f;   // the experts this handle holds
    // canonical layout (the fused launch), and the tiled copies as
    // [rows x k-blocks][128 bytes]: box (0, tiled_row(...)) of 256 (or 128) rows
    // is one k-block of a tile (or half of it)
    const uint64_t gu_rows = E * 2 * f * (d / BK), dn_rows = E * d * (f / BK);
    return make_map(&w->tm_w_gu, w->w_gu, d, E * 2 * f, BN) && make_map(&w->tm_w_dn, w->w_dn, f, E * d, BN) &&
           w->w_gu_t && w->w_dn_t &&
           make_map(&w->tm_w_gu_t, w->w_gu_t, BK, gu_rows, BN) && make_map(&w->tm_w_dn_t, w->w_dn_t, BK, dn_rows, BN) &&
           make_map(&w->tm_w_gu_t_half, w->w_gu_t, BK, gu_rows, BN / 2) &&
           make_map(&w->tm_w_dn_t_half, w->w_dn_t, BK, dn_rows, BN / 2);
}

namespace {
// One 32 KB chunk (256 rows x 128 bytes) per block: thread r copies row r's
// 128 bytes of k-block kb.
__global__ void __launch_bounds__(256) tile_weights_kernel(const int8_t* __restrict__ src, int K,
                                                           int8_t* __restrict__ dst) {
    const int nkb = K / BK;
    const int64_t chunk = blockIdx.x;
    const int64_t rt = chunk / nkb;
    const int kb = (int)(chunk % nkb), r = threadIdx.x;
    const int4* in = reinterpret_cast<const int4*>(src + (rt * BN + r) * (int64_t)K + kb * BK);
    int4* out = reinterpret_cast<int4*>(dst + (chunk * BN + r) * BK);
#pragma unroll
    for (int j = 0; j < BK / 16; ++j) out[j] = in[j];
}
}  // namespace

cudaError_t launch_tile_weights(const int8_t* src, int64_t rows, int K, int8_t* dst, cudaStream_t s) {
    if (rows % BN || K % BK) return cudaErrorInvalidValue;
    const int64_t chunks = rows / BN * (K / BK);
    if (chunks > INT32_MAX) return cudaErrorInvalidValue;
    tile_weights_kernel<<<(unsigned)chunks, 256, 0, s>>>(src, K, dst);
    return cudaGetLastError();
}

template <int FMT, bool SW>
cudaError_t launch_fused_fmt(const CUtensorMap& a1, const CUtensorMap& b1, const CUtensorMap& a2,
                             const CUtensorMap& b2, const TcParams& p1, const TcParams& p2, const FusedExtra& fx,
                             int grid, cudaStream_t s) {
    static std::atomic<uint64_t> attr{0};
    constexpr size_t smem = FusedPlan<SW>::kSmem;
    cudaError_t e = smem_attr_once(tc_ffn_fused_kernel<FMT, SW>, smem, attr);
    if (e != cudaSuccess) return e;
    return launch_pdl(tc_ffn_fused_kernel<FMT, SW>, dim3(grid), dim3(kFusedThreads), smem, s, a1, b1, a2, b2, p1,
                      p2, fx);
}

cudaError_t launch_tc_ffn_fused(const moe_w8a8_weights* w, int T, const int8_t* aq, const int32_t* meta,
                                const int32_t* tiles, const int32_t* offsets, const int32_t* row2ts,
                                const float* sx, const float* topk_w, float* h32, float* pamax, int8_t* hq,
                                float* sh, void* o, int32_t* acc1_dbg, int32_t* acc2_dbg, int32_t* sync_words,
                                cudaStream_t s) {
    const moe_w8a8_config& c = w->cfg;
    const int rows = T * c.top_k;
    CUtensorMap a1, a2;
    // at most kFusedSwapRows tokens: each m-tile holds at most that many rows (a token
    // adds at most one row per expert), and the swapped-operand plan runs
    const bool sw = fused_swapped(T);
    const uint32_t trows = sw ? kFusedSwapRows : BM;
    if (!make_map(&a1, aq, c.d, rows, trows) || !make_map(&a2, hq, c.f, rows, trows)) return cudaErrorInvalidValue;
    TcParams p1{}, p2{};
    p1.N = 2 * c.f;
    p1.K = c.d;
    p1.n_tiles_n = p1.N / BN;
    p2.N = c.d;
    p2.K = c.f;
    p2.n_tiles_n = p2.N / BN;
    for (TcParams* p : {&p1, &p2}) {
        p->f = c.f;
        p->k = c.top_k;
        p->meta = meta;
        p->tiles = tiles;
        p->offsets = offsets;
        p->row2ts = row2ts;
        p->status = w->status;
    }
    p1.sx = sx;
    p1.sw0 = w->sw_gate;
    p1.sw1 = w->sw_up;
    p1.h32 = h32;
    p1.pamax = pamax;
    p1.acc_dbg = acc1_dbg;
    p2.topk_w = topk_w;
    p2.sw0 = w->sw_dn;
    p2.sh = sh;
    p2.o = o;
    p2.o_bf16 = c.out_dtype == MOE_BF16;
    p2.acc_dbg = acc2_dbg;
    const int max_mt = (rows + BM - 1) / BM + c.n_experts;
    const FusedExtra fx{sync_words, sync_words + max_mt, sync_words + 2 * max_mt, sync_words + 2 * max_mt + 1, hq,
                        sh, w->wait_budget_ns, w->test_skip_ready};
    const int grid = max(1, min(w->num_sms, max_mt * (p1.n_tiles_n + p2.n_tiles_n)));
    if (c.expert_format == FMT_E4M3)
        return sw ? launch_fused_fmt<FMT_E4M3, true>(a1, w->tm_w_gu, a2, w->tm_w_dn, p1, p2, fx, grid, s)
                  : launch_fused_fmt<FMT_E4M3, false>(a1, w->tm_w_gu, a2, w->tm_w_dn, p1, p2, fx, grid, s);
    return sw ? launch_fused_fmt<FMT_INT8, true>(a1, w->tm_w_gu, a2, w->tm_w_dn, p1, p2, fx, grid, s)
              : launch_fused_fmt<FMT_INT8, false>(a1, w->tm_w_gu, a2, w->tm_w_dn, p1, p2, fx, grid, s);
}

bool router_tc_make_maps(moe_w8a8_weights* w) {
    return make_map_bf16(&w->tm_rt_hi, w->rt_hi, w->cfg.d, w->rt_epad, kRcSlice) &&
           make_map_bf16(&w->tm_rt_lo, w->rt_lo, w->cfg.d, w->rt_epad, kRcSlice);
}

cudaError_t launch_router_tc(const moe_w8a8_weights* w, const void* x, int T, float* approx, cudaStream_t s) {
    CUtensorMap mx;
    if (!make_map_bf16(&mx, x, w->cfg.d, T, BM)) return cudaErrorInvalidValue;
    // 64 experts per CTA whatever the padded count: more CTAs for wide routers
    if (w->rt_epad % kRcSlice) return cudaErrorInvalidValue;
    return launch_router_tc_pad<kRcSlice>(mx, w, T, approx, s);
}

cudaError_t launch_tc_peak(int fmt, int64_t n_mma, int grid, cudaStream_t s) {
    static std::atomic<uint64_t> a8{0}, af8{0};
    if (fmt == FMT_E4M3) {
        cudaError_t e = smem_attr_once(tc_peak_kernel<FMT_E4M3>, kPeakSmem, af8);
        if (e != cudaSuccess) return e;
        return launch_pdl(tc_peak_kernel<FMT_E4M3>, dim3(grid), dim3(kPeakThreads), kPeakSmem, s, n_mma);
    }
    cudaError_t e = smem_attr_once(tc_peak_kernel<FMT_INT8>, kPeakSmem, a8);
    if (e != cudaSuccess) return e;
    return launch_pdl(tc_peak_kernel<FMT_INT8>, dim3(grid), dim3(kPeakThreads), kPeakSmem, s, n_mma);
}

bool tc_supported(const moe_w8a8_config& c) { return c.d % BN == 0 && c.f % BK == 0 && c.d % BK == 0; }

cudaError_t launch_requant(const float* h32, const float* pamax, int f, const int32_t* meta,
                           int max_rows, int8_t* hq, float* sh, int fmt, cudaStream_t s) {
    const int rows_per_block = kRqThreads / 32;
    const dim3 grid((max_rows + rows_per_block - 1) / rows_per_block);
    if (fmt == FMT_E4M3)
        return launch_pdl(requant_kernel<FMT_E4M3>, grid, dim3(kRqThreads), 0, s, h32, pamax, f, meta, hq, sh);
    return launch_pdl(requant_kernel<FMT_INT8>, grid, dim3(kRqThreads), 0, s, h32, pamax, f, meta, hq, sh);
}

cudaError_t launch_tc_gemm1(const moe_w8a8_weights* w, int T, const int8_t* aq, const int32_t* meta,
                            const int32_t* tiles, const int32_t* pairs, const int32_t* offsets,
                            const int32_t* row2ts, const float* sx, float* h32, float* pamax, int32_t* acc_dbg,
                            cudaStream_t s) {
    const moe_w8a8_config& c = w->cfg;
    CUtensorMap ta;
    const int rows = T * c.top_k;
    if (!make_map(&ta, aq, c.d, rows, BM)) return cudaErrorInvalidValue;
    TcParams p{};
    p.N = 2 * c.f;
    p.K = c.d;
    p.n_tiles_n = p.N / BN;
    p.f = c.f;
    p.k = c.top_k;
    p.meta = meta;
    p.tiles = tiles;
    p.offsets = offsets;
    p.row2ts = row2ts;
    p.sx = sx;
    p.sw0 = w->sw_gate;
    p.sw1 = w->sw_up;
    p.h32 = h32;
    p.pamax = pamax;
    p.acc_dbg = acc_dbg;
    p.status = w->status;
    p.pairs = pairs;
    CUtensorMap tc;
    if (!make_out_map(&tc, h32, c.f, rows, false)) return cudaErrorInvalidValue;
    p.tma_c = 1;
    if (pairs) {
        const int max_pt = (rows + 2 * BM - 1) / (2 * BM) + w->n_local;
        return launch_pair<EPI_SWIGLU>(ta, w->tm_w_gu_t_half, tc, p, max_pt * p.n_tiles_n, c.expert_format, s);
    }
    const int max_mt = (rows + BM - 1) / BM + c.n_experts;
    const int grid = max(1, min(w->num_sms, max_mt * p.n_tiles_n));
    return launch<EPI_SWIGLU>(ta, w->tm_w_gu_t, tc, p, grid, c.expert_format, s);
}

cudaError_t launch_tc_gemm2(const moe_w8a8_weights* w, int T, const int8_t* hq, const float* sh,
                            const int32_t* meta, const int32_t* tiles, const int32_t* pairs,
                            const int32_t* offsets, const int32_t* row2ts, const float* topk_w, void* o,
                            int32_t* acc_dbg, cudaStream_t s) {
    const moe_w8a8_config& c = w->cfg;
    CUtensorMap ta;
    const int rows = T * c.top_k;
    if (!make_map(&ta, hq, c.f, rows, BM)) return cudaErrorInvalidValue;
    TcParams p{};
    p.N = c.d;
    p.K = c.f;
    p.n_tiles_n = p.N / BN;
    p.f = c.f;
    p.k = c.top_k;
    p.meta = meta;
    p.tiles = tiles;
    p.offsets = offsets;
    p.row2ts = row2ts;
    p.topk_w = topk_w;
    p.sw0 = w->sw_dn;
    p.sh = sh;
    p.o = o;
    p.o_bf16 = c.out_dtype == MOE_BF16;
    p.acc_dbg = acc_dbg;
    p.status = w->status;
    p.pairs = pairs;
    // bf16 O rows leave through bulk tensor stores; fp32 rows (128 bytes per
    // chunk row) keep the plain stores, and the map is then only a placeholder
    CUtensorMap tc;
    if (!make_out_map(&tc, o, c.d, rows, true)) return cudaErrorInvalidValue;
    p.tma_c = p.o_bf16;
    if (pairs) {
        const int max_pt = (rows + 2 * BM - 1) / (2 * BM) + w->n_local;
        return launch_pair<EPI_DOWN>(ta, w->tm_w_dn_t_half, tc, p, max_pt * p.n_tiles_n, c.expert_format, s);
    }
    const int max_mt = (rows + BM - 1) / BM + c.n_experts;
    const int grid = max(1, min(w->num_sms, max_mt * p.n_tiles_n));
    return launch<EPI_DOWN>(ta, w->tm_w_dn_t, tc, p, grid, c.expert_format, s);
}

}  // namespace moe
