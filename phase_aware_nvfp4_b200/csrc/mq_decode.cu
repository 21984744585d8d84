// mq_decode.cu -- the precise decode path: BF16 GEMV / skinny GEMM on the
// BF16 master weights, FP32 accumulation ("Mix-Quant: Quantized Prefilling,
// Precise Decoding for Agentic LLMs", section 3.3, "Prefill-Decode
// Disaggregation Deployment": the decode path keeps the original
// high-precision weights; section 3.1: decoding is bound by memory access).
//
// Y[M, N] = X[M, K] W[N, K]^T with M <= 256 tokens.  The kernel computes the
// transposed product on the tensor cores, D[n, m] = sum_k W[n, k] X[m, k]:
// A = a 128-row W tile streamed by TMA, B = the (zero-padded) token tile,
// D = 128 lanes x MT columns of FP32 in TMEM.  The W stream is the whole
// cost, so the grid must cover every SM: the K dimension is split across the
// CTAs of a thread-block cluster and the partial sums are reduced through
// distributed shared memory (no global scratch, deterministic order).
#include <map>
#include <mutex>
#include <tuple>

#include "mq_device.cuh"

namespace mq {
namespace {

constexpr int DBM = 128;                 // W rows per tile (UMMA M)
constexpr int DBK = 64;                  // K elements per stage (128 bytes of BF16)
constexpr int D_THREADS = 192;
constexpr int W_STAGE = DBM * DBK * 2;   // 16 KiB

// NVFP4 weights (FMT 1): 256 K-elements per stage = 128 bytes of codes per
// row, plus four 512-byte scale atoms for the 128 W rows and four for the
// (at most 128) tokens.
constexpr int QBK = 256;
constexpr int QW_CODES = DBM * QBK / 2;   // 16 KiB
constexpr int Q_SF = 4 * 512;             // 2 KiB

struct DParams {
    int M, N, K, MT;
    int k_stages;       // total K stages
    int split;          // cluster size along K
    int stages;         // pipeline depth
    int stage_bytes;
    int bar_offset;     // barriers sit after both the pipeline and the partial-sum buffer
    uint32_t tmem_cols;
    uint32_t tmem_sf;   // FMT 1: first TMEM column of the scale factors (A at +0, B at +16)
    int sfw_atoms, sfx_atoms;   // FMT 1: scale atoms per 128-row block of W and of X
    const float* alpha_w;       // FMT 1: tensor scales
    const float* alpha_x;
    uint16_t* y;
    WsControl* ctrl;
};

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_addr, uint32_t rank)
{
    uint32_t raddr;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(local_addr), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(raddr) : "memory");
    return v;
}

// FMT 0: W and X BF16, kind::f16, 64 K-elements per stage.
// FMT 1: W and X NVFP4 (codes + E4M3 block scales + FP32 tensor scales),
//        kind::mxf4nvf4 block-scaled MMAs, 256 K-elements per stage; the
//        scale atoms are copied SMEM -> TMEM per 64-element k-block and
//        the result is scaled by fl(alpha_w * alpha_x).
// Stage layout: [W tile][X tile] (both 128-byte-swizzled, 1024-aligned),
// then for FMT 1 [W scale atoms][X scale atoms].
template <int FMT>
__global__ void __launch_bounds__(D_THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                  const __grid_constant__ CUtensorMap tmap_sfw, const __grid_constant__ CUtensorMap tmap_sfx,
                  const DParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int W_TILE = FMT ? QW_CODES : W_STAGE;
    const int x_tile = FMT ? p.MT * (QBK / 2) : p.MT * DBK * 2;
    const int stage_bytes = p.stage_bytes;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + p.bar_offset);
    uint64_t* empty_bar = full_bar + p.stages;
    uint64_t* acc_full = empty_bar + p.stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    float* red = reinterpret_cast<float*>(smem);  // [MT][128] partials, reuses the pipeline buffers

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = (p.split > 1) ? cluster_rank() : 0u;
    const int n_tile = blockIdx.x / p.split;
    const int ks_begin = (int)(((int64_t)p.k_stages * rank) / p.split);
    const int ks_end = (int)(((int64_t)p.k_stages * (rank + 1)) / p.split);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&tmap_w);
        prefetch_tensormap(&tmap_x);
        if (FMT) {
            prefetch_tensormap(&tmap_sfw);
            prefetch_tensormap(&tmap_sfx);
        }
    }
    if (warp == 1) tmem_alloc(tmem_slot, p.tmem_cols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // TMA producer: whole warp (warp-uniform values), one elected lane issues
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int last_stage = -1;
        uint32_t last_parity = 0;
        int ks = ks_begin;
        if (FMT) {
            // The tokens and alpha_x come from the quantization kernel just
            // before this one (programmatic dependent launch): fill the first
            // ring slots with weight tiles and scales, wait for that kernel,
            // then add the token tiles to those slots.
            const int pre = std::min(p.stages, ks_end - ks_begin);
            if (elect_one()) {
                for (int i = 0; i < pre; ++i) {
                    uint8_t* sw = smem + i * stage_bytes;
                    mbar_arrive_expect_tx(&full_bar[i], (uint32_t)stage_bytes);
                    tma_load_2d(sw, &tmap_w, &full_bar[i], (ks_begin + i) * (QBK / 2), n_tile * DBM);
                    tma_load_2d(sw + W_TILE + x_tile, &tmap_sfw, &full_bar[i], 0,
                                n_tile * p.sfw_atoms + (ks_begin + i) * 4);
                }
            }
            __syncwarp();
            grid_dep_wait();
            if (elect_one()) {
                for (int i = 0; i < pre; ++i) {
                    uint8_t* sw = smem + i * stage_bytes;
                    tma_load_2d(sw + W_TILE, &tmap_x, &full_bar[i], (ks_begin + i) * (QBK / 2), 0);
                    tma_load_2d(sw + W_TILE + x_tile + Q_SF, &tmap_sfx, &full_bar[i], 0, (ks_begin + i) * 4);
                }
            }
            __syncwarp();
            if (pre > 0) {
                last_stage = pre - 1;
                last_parity = 0;
            }
            ks += pre;
            stage = pre;
            if (stage == p.stages) stage = 0, phase = 1u;
        }
        for (; ks < ks_end; ++ks) {
            if (!warp_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (elect_one()) {
                mbar_arrive_expect_tx(&full_bar[stage], (uint32_t)stage_bytes);
                uint8_t* sw = smem + stage * stage_bytes;
                if (FMT) {
                    // codes: x = byte column; scales: 4 atoms of this stage
                    tma_load_2d(sw, &tmap_w, &full_bar[stage], ks * (QBK / 2), n_tile * DBM);
                    tma_load_2d(sw + W_TILE, &tmap_x, &full_bar[stage], ks * (QBK / 2), 0);
                    tma_load_2d(sw + W_TILE + x_tile, &tmap_sfw, &full_bar[stage], 0, n_tile * p.sfw_atoms + ks * 4);
                    tma_load_2d(sw + W_TILE + x_tile + Q_SF, &tmap_sfx, &full_bar[stage], 0, ks * 4);
                } else {
                    tma_load_2d(sw, &tmap_w, &full_bar[stage], ks * DBK, n_tile * DBM);
                    tma_load_2d(sw + W_TILE, &tmap_x, &full_bar[stage], ks * DBK, 0);
                }
            }
            __syncwarp();
            last_stage = stage;
            last_parity = phase;
            if (++stage == p.stages) stage = 0, phase ^= 1u;
        }
        if (!ok) {
            if (lane == 0) {
                post_error(p.ctrl, kErrTimeout);
                *abort_flag = 1;
            }
            // stages are consumed in order, so the newest issue lands last
            if (last_stage >= 0) (void)mbar_wait(&full_bar[last_stage], last_parity);
        }
    } else if (warp == 1) {
        // MMA issuer: whole warp, one elected lane issues
        const uint32_t idesc = FMT ? idesc_nvfp4(DBM, p.MT) : idesc_bf16(DBM, p.MT);
        const uint64_t w_desc0 = sdesc_kmajor_sw128(smem_u32(smem));
        const uint64_t sf_desc0 = sdesc_sf_block(smem_u32(smem + W_TILE + x_tile));
        const uint32_t sfa_tmem = tmem_base + p.tmem_sf;
        const uint32_t sfb_tmem = sfa_tmem + 16;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true, next_ready = false;
        for (int ks = ks_begin; ks < ks_end; ++ks) {
            if (!next_ready && !warp_wait(&full_bar[stage], phase, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            {   // look at the next ring stage now; its result is used next iteration
                const int ns = (stage + 1 == p.stages) ? 0 : stage + 1;
                next_ready = warp_test(&full_bar[ns], ns == 0 ? (phase ^ 1u) : phase);
            }
            const uint64_t w_d = w_desc0 + (uint64_t)((stage * stage_bytes) >> 4);
            const uint64_t x_d = w_d + (uint64_t)(W_TILE >> 4);
            const uint64_t sf_d = sf_desc0 + (uint64_t)((stage * stage_bytes) >> 4);
            if (elect_one()) {
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    const uint32_t acc = (ks > ks_begin || kb > 0) ? 1u : 0u;
                    if (FMT) {
                        tmem_cp_32x128b_x4(sfa_tmem + 4 * kb, sf_d + (uint64_t)((kb * 512) >> 4));
                        tmem_cp_32x128b_x4(sfb_tmem + 4 * kb, sf_d + (uint64_t)((Q_SF + kb * 512) >> 4));
                        umma_nvfp4(tmem_base, w_d + (uint64_t)((32 * kb) >> 4), x_d + (uint64_t)((32 * kb) >> 4), idesc,
                                   sfa_tmem + 4 * kb, sfb_tmem + 4 * kb, acc);
                    } else {
                        umma_bf16(tmem_base, w_d + (uint64_t)((32 * kb) >> 4), x_d + (uint64_t)((32 * kb) >> 4), idesc,
                                  acc);
                    }
                }
                tc_commit(&empty_bar[stage]);
            }
            __syncwarp();
            if (++stage == p.stages) stage = 0, phase ^= 1u;
        }
        if (!ok && lane == 0) {
            post_error(p.ctrl, kErrTimeout);
            *abort_flag = 1;
        }
        if (elect_one()) tc_commit(acc_full);  // also the "all MMAs done" signal before TMEM is freed
        __syncwarp();
    } else {
        const int lg = warp & 3;
        const int row = 32 * lg + lane;  // W row within the tile = TMEM lane
        const int64_t n = (int64_t)n_tile * DBM + row;
        const bool have_acc = ks_end > ks_begin;
        // FMT 1 output scale fl(alpha_w * alpha_x), applied to the FP32 sum;
        // alpha_x is written by the preceding kernel
        if (FMT) grid_dep_wait();
        const float out_scale = FMT ? __fmul_rn(*p.alpha_w, *p.alpha_x) : 1.0f;
        bool ok = mbar_wait(acc_full, 0);
        if (!ok) post_error(p.ctrl, kErrTimeout);
        tc_fence_after();
        const uint32_t t_row = tmem_base + ((uint32_t)(32 * lg) << 16);
        for (int c = 0; c < p.MT / 16; ++c) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(t_row + 16 * c, r);
            tmem_wait_ld(r);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int m = 16 * c + j;
                const float v = (have_acc && ok) ? __uint_as_float(r[j]) : 0.0f;
                if (p.split > 1) {
                    red[m * DBM + row] = v;
                } else if (m < p.M && n < p.N) {
                    const float o = FMT ? __fmul_rn(v, out_scale) : v;
                    p.y[(int64_t)m * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
                }
            }
        }
    }

    if (p.split > 1) {
        // Every CTA of the cluster has its partial tile in shared memory; CTA
        // `rank` reduces tokens m = rank, rank + split, ... in rank order.
        cluster_sync_all();
        if (warp >= 2) {
            const int row = 32 * (warp & 3) + lane;
            const int64_t n = (int64_t)n_tile * DBM + row;
            const float out_scale = FMT ? __fmul_rn(*p.alpha_w, *p.alpha_x) : 1.0f;
            for (int m = (int)rank; m < p.M; m += p.split) {
                float acc = 0.0f;
                const uint32_t laddr = smem_u32(&red[m * DBM + row]);
                for (int q = 0; q < p.split; ++q) acc += ld_dsmem_f32(laddr, (uint32_t)q);
                if (FMT) acc = __fmul_rn(acc, out_scale);
                if (n < p.N) p.y[(int64_t)m * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
            }
        }
        cluster_sync_all();  // keep every partial alive until all readers are done
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

// CTAs of decode_kernel<FMT> that can be resident at once when launched in
// clusters of `cluster` CTAs with `smem` bytes of dynamic shared memory.
template <int FMT>
int max_resident_ctas(int cluster, int smem, const DeviceInfo& di)
{
    static std::mutex mu;
    static std::map<std::tuple<int, int, int>, int> cache;
    const auto key = std::make_tuple(di.device, cluster, smem);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    auto kern = decode_kernel<FMT>;
    int ctas = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
        if (cluster == 1) {
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, D_THREADS, smem) == cudaSuccess)
                ctas = per_sm * di.num_sms;
        } else {
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3((unsigned)(cluster * di.num_sms), 1, 1);
            cfg.blockDim = dim3(D_THREADS, 1, 1);
            cfg.dynamicSmemBytes = (size_t)smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)cluster;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess) ctas = clusters * cluster;
        }
    }
    (void)cudaGetLastError();   // a failed query is not an error of the caller's stream
    cache[key] = ctas;
    return ctas;
}

// Launch shape.  W streams from HBM, so what matters is how many bytes are in
// flight: about kSaturateBytes over the whole GPU keep HBM busy.  Candidates:
// K split (= cluster size) a power of two <= 8, with either a shallow
// pipeline (~100 KB, two CTAs per SM) or a deep one (~200 KB, one CTA per
// SM).  How many clusters of a size can be resident depends on how they pack
// into the GPCs, so that is asked of the runtime (cached).  A candidate must
// run in one wave; the most bytes in flight (capped at the saturation point)
// wins, then the larger grid, then the smaller split and the shallow pipeline.  Fills split,
// stages, bar_offset; returns the dynamic shared memory size.
template <int FMT>
int choose_shape(DParams& p, int n_tiles, const DeviceInfo& di)
{
    constexpr int64_t kSaturateBytes = 16ll << 20;
    const int stage_bytes = p.stage_bytes;
    const int red_bytes = p.MT * DBM * 4;
    int best_split = 1, best_stages = std::max(2, std::min(8, 100 * 1024 / stage_bytes));
    int64_t best_score = -1;
    for (int sp = 1; sp <= 8 && sp <= p.k_stages; sp *= 2) {
        const int per_cta_stages = (p.k_stages + sp - 1) / sp;
        for (int deep = 0; deep < 2; ++deep) {
            int st = deep ? std::min(12, 200 * 1024 / stage_bytes) : std::min(8, 100 * 1024 / stage_bytes);
            st = std::max(2, std::min(st, std::max(2, per_cta_stages)));
            const int sm = std::max(st * stage_bytes, red_bytes) + 256 + 1024;
            if ((size_t)sm > di.max_smem_optin) continue;
            const int active = max_resident_ctas<FMT>(sp, sm, di);
            const int ctas = n_tiles * sp;
            if (active <= 0 || ctas > active) continue;
            // a CTA streams at a bounded rate, so once the bytes in flight are
            // saturated more CTAs still help: ties go to the larger grid
            const int64_t score = std::min<int64_t>(kSaturateBytes, (int64_t)ctas * st * stage_bytes) * 1024 +
                                  std::min(ctas, 1023);
            if (score > best_score) {
                best_score = score;
                best_split = sp;
                best_stages = st;
            }
        }
    }
    p.split = best_split;
    p.stages = best_stages;
    p.bar_offset = std::max(p.stages * stage_bytes, red_bytes);
    return p.bar_offset + 256 + 1024;
}

template <int FMT>
cudaError_t launch_shape(const DParams& p, int n_tiles, int smem, const CUtensorMap& tw, const CUtensorMap& tx,
                         const CUtensorMap& tsfw, const CUtensorMap& tsfx, cudaStream_t s)
{
    auto kern = decode_kernel<FMT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(n_tiles * p.split), 1, 1);
    cfg.blockDim = dim3(D_THREADS, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p.split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // FMT 1 follows the token quantization on the stream: let it start early
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = FMT ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, tw, tx, tsfw, tsfx, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_bf16(const void* x, int64_t M, const void* w, int64_t N, int64_t K, void* y,
                               WsControl* ctrl, const DeviceInfo& di, cudaStream_t s)
{
    DParams p{};
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.MT = (int)((M + 15) / 16 * 16);
    p.k_stages = (int)((K + DBK - 1) / DBK);
    p.tmem_cols = 32;
    while ((int)p.tmem_cols < p.MT) p.tmem_cols <<= 1;
    p.y = static_cast<uint16_t*>(y);
    p.ctrl = ctrl;
    p.stage_bytes = W_STAGE + p.MT * DBK * 2;
    const int n_tiles = (int)((N + DBM - 1) / DBM);
    const int smem = choose_shape<0>(p, n_tiles, di);

    CUtensorMap tw, tx;
    if (!make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, DBK, DBM,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, DBK,
                      (uint32_t)p.MT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    return launch_shape<0>(p, n_tiles, smem, tw, tx, tw, tx, s);
}

cudaError_t launch_decode_nvfp4(const uint8_t* x_codes, const uint8_t* x_scales, const float* alpha_x, int64_t M,
                                const uint8_t* w_codes, const uint8_t* w_scales, const float* alpha_w, int64_t N,
                                int64_t K, void* y, WsControl* ctrl, const DeviceInfo& di, cudaStream_t s)
{
    DParams p{};
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.MT = (int)((M + 31) / 32 * 32);   // MMA N: a multiple of 32, at most 128
    p.k_stages = (int)((K + QBK - 1) / QBK);
    uint32_t acc_cols = 32;
    while ((int)acc_cols < p.MT) acc_cols <<= 1;
    p.tmem_sf = acc_cols;                // A scales at +0..15, B scales at +16..31
    p.tmem_cols = 32;
    while (p.tmem_cols < acc_cols + 32) p.tmem_cols <<= 1;
    p.sfw_atoms = (int)sf_atoms_per_rowblk(K);
    p.sfx_atoms = (int)sf_atoms_per_rowblk(K);
    p.alpha_w = alpha_w;
    p.alpha_x = alpha_x;
    p.y = static_cast<uint16_t*>(y);
    p.ctrl = ctrl;
    p.stage_bytes = QW_CODES + p.MT * (QBK / 2) + 2 * Q_SF;
    const int n_tiles = (int)((N + DBM - 1) / DBM);
    const int smem = choose_shape<1>(p, n_tiles, di);

    CUtensorMap tw, tx, tsfw, tsfx;
    if (!make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, (uint64_t)(K / 2), (uint64_t)N, (uint64_t)(K / 2),
                      QBK / 2, DBM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, x_codes, (uint64_t)(K / 2), (uint64_t)M, (uint64_t)(K / 2),
                      QBK / 2, (uint32_t)p.MT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    // scale buffers viewed as rows of one 512-byte atom (128 x u32); a box is 4 atoms
    if (!make_tmap_2d(&tsfw, CU_TENSOR_MAP_DATA_TYPE_UINT32, w_scales, 128,
                      (uint64_t)sf_rowblks(N) * (uint64_t)p.sfw_atoms, 512, 128, 4, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tsfx, CU_TENSOR_MAP_DATA_TYPE_UINT32, x_scales, 128,
                      (uint64_t)sf_rowblks(M) * (uint64_t)p.sfx_atoms, 512, 128, 4, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    return launch_shape<1>(p, n_tiles, smem, tw, tx, tsfw, tsfx, s);
}

}  // namespace mq
