// mq_decode.cu -- the precise decode path: BF16 GEMV / skinny GEMM on the
// BF16 master weights, FP32 accumulation ("Mix-Quant: Quantized Prefilling,
// Precise Decoding for Agentic LLMs", section 3.3, "Prefill-Decode
// Disaggregation Deployment": the decode path keeps the original
// high-precision weights; section 3.1: decoding is bound by memory access).
//
// Y[M, N] = X[M, K] W[N, K]^T with M <= 256 tokens.  A single token runs on
// the CUDA cores (decode_gemv_kernel).  Otherwise the kernel computes the
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
constexpr int DBK = 64;                  // K elements per TMA box (128 bytes of BF16)
constexpr int D_THREADS = 192;
constexpr int W_STAGE = DBM * DBK * 2;   // 16 KiB per box

// NVFP4 weights (FMT 1): 256 K-elements per stage = 128 bytes of codes per
// row, plus four 512-byte scale atoms for the 128 W rows and four for the
// (at most 128) tokens.
constexpr int QBK = 256;
constexpr int QW_CODES = DBM * QBK / 2;   // 16 KiB
constexpr int Q_SF = 4 * 512;             // 2 KiB

struct DParams {
    int M, N, K, MT;
    int k_stages;       // total K stages
    int kbox;           // FMT 0: TMA boxes of DBK elements per stage (one wait, commit and
                        // hand-over per stage: larger stages issue fewer of them per byte)
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
    // K split across independent CTAs (gpart != 0) instead of a cluster: each
    // writes its FP32 partial tile to `part`, the last of a tile's CTAs (by
    // the per-tile counter) adds them in rank order and writes Y
    int gpart;
    float* part;
    uint32_t* tile_ctr;
};

constexpr int kDecodeMaxSplit = 8;        // CTAs per 128-row tile in the split-K through the workspace
constexpr int kDecodeMaxGpartTokens = 16; // tokens up to which that split is used (its reduction is serial per tile)

// Split-K reduction through global memory for one 128-row decode tile, run by
// the 128 epilogue threads (named barrier 2; `row` = TMEM lane = W row of the
// tile).  Every CTA of the tile has stored its partial part[tile][rank][m][row]
// for m < M; the CTA that takes the last ticket of the tile's counter adds
// the `split` partials in rank order (so the result does not depend on which
// CTA finishes last), scales by out_scale and writes Y[m][n] in BF16, and
// resets the counter for the next call.
__device__ __forceinline__ void gsplit_reduce(float* part, uint32_t* tile_ctr, uint32_t* s_flag, int tile, int split,
                                              int M, int N, int row, int lead, float out_scale, uint16_t* y)
{
    // every thread's partial stores precede the lead's ticket, whose release
    // covers them; the last CTA's threads read after its acquire
    named_barrier_sync(2, 128);
    if (lead) *s_flag = (atom_add_acq_rel_gpu(&tile_ctr[tile], 1u) == (uint32_t)(split - 1)) ? 1u : 0u;
    named_barrier_sync(2, 128);
    if (*s_flag == 0u) return;
    const int64_t n = (int64_t)tile * DBM + row;
    const float* base = part + (int64_t)tile * split * M * DBM + row;
    for (int m0 = 0; m0 < M; m0 += 4) {
        // the partials of four tokens from all splits in flight at once, then
        // each token's sum in rank order
        float v[4][kDecodeMaxSplit];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int q = 0; q < kDecodeMaxSplit; ++q)
                v[t][q] = (m0 + t < M && q < split) ? __ldcg(base + ((int64_t)q * M + m0 + t) * DBM) : 0.0f;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float acc = 0.0f;
#pragma unroll
            for (int q = 0; q < kDecodeMaxSplit; ++q)
                if (q < split) acc += v[t][q];
            if (m0 + t < M && n < N)
                y[(int64_t)(m0 + t) * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(acc, out_scale)));
        }
    }
    if (lead) tile_ctr[tile] = 0u;
}

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
    const int W_TILE = FMT ? QW_CODES : W_STAGE * p.kbox;
    const int x_box = p.MT * DBK * 2;   // FMT 0: bytes of one token box
    const int x_tile = FMT ? p.MT * (QBK / 2) : x_box * p.kbox;
    const int stage_bytes = p.stage_bytes;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + p.bar_offset);
    uint64_t* empty_bar = full_bar + p.stages;
    uint64_t* acc_full = empty_bar + p.stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    uint32_t* s_last = tmem_slot + 2;
    float* red = reinterpret_cast<float*>(smem);  // [MT][128] partials, reuses the pipeline buffers

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = (p.split > 1) ? (p.gpart ? (uint32_t)(blockIdx.x % p.split) : cluster_rank()) : 0u;
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
    // BF16 path: the previous kernel of the stream may have written X, W or Y.
    // (The NVFP4 path waits where it first reads what its predecessor, the
    // token quantization, wrote.)
    if (!FMT) {
        grid_dep_wait();
        grid_dep_launch_dependents();
    }

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
                    for (int b = 0; b < p.kbox; ++b) {
                        const int kx = (ks * p.kbox + b) * DBK;   // boxes past K read zeros
                        tma_load_2d(sw + b * W_STAGE, &tmap_w, &full_bar[stage], kx, n_tile * DBM);
                        tma_load_2d(sw + W_TILE + b * x_box, &tmap_x, &full_bar[stage], kx, 0);
                    }
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
                if (FMT) {
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        const uint32_t acc = (ks > ks_begin || kb > 0) ? 1u : 0u;
                        tmem_cp_32x128b_x4(sfa_tmem + 4 * kb, sf_d + (uint64_t)((kb * 512) >> 4));
                        tmem_cp_32x128b_x4(sfb_tmem + 4 * kb, sf_d + (uint64_t)((Q_SF + kb * 512) >> 4));
                        umma_nvfp4(tmem_base, w_d + (uint64_t)((32 * kb) >> 4), x_d + (uint64_t)((32 * kb) >> 4), idesc,
                                   sfa_tmem + 4 * kb, sfb_tmem + 4 * kb, acc);
                    }
                } else {
                    for (int b = 0; b < p.kbox; ++b) {
                        const uint64_t wb = w_d + (uint64_t)((b * W_STAGE) >> 4);
                        const uint64_t xb = x_d + (uint64_t)((b * x_box) >> 4);
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb)
                            umma_bf16(tmem_base, wb + (uint64_t)((32 * kb) >> 4), xb + (uint64_t)((32 * kb) >> 4),
                                      idesc, (ks > ks_begin || b > 0 || kb > 0) ? 1u : 0u);
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
                if (p.split > 1 && p.gpart) {
                    if (m < p.M) p.part[(((int64_t)n_tile * p.split + rank) * p.M + m) * DBM + row] = v;
                } else if (p.split > 1) {
                    red[m * DBM + row] = v;
                } else if (m < p.M && n < p.N) {
                    const float o = FMT ? __fmul_rn(v, out_scale) : v;
                    p.y[(int64_t)m * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
                }
            }
        }
        if (p.split > 1 && p.gpart)
            gsplit_reduce(p.part, p.tile_ctr, s_last, n_tile, p.split, p.M, p.N, row, warp == 2 && lane == 0,
                          FMT ? out_scale : 1.0f, p.y);
    }

    if (p.split > 1 && !p.gpart) {
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

// Bytes of shared memory that keep the CTAs sharing an SM within its 512 TMEM
// columns (each CTA allocates tmem_cols): smem is padded so that at most
// 512 / tmem_cols CTAs fit.
inline int pad_smem_for_tmem(int smem, uint32_t tmem_cols, const DeviceInfo& di)
{
    const int cap = 512 / (int)tmem_cols;
    const int per_sm_min = (int)(di.smem_per_sm / (size_t)(cap + 1)) + 1;   // bytes incl. the runtime's reserve
    smem = std::max<int>(smem, per_sm_min - (int)di.smem_reserved_per_cta);
    return (smem + 1023) / 1024 * 1024;
}

// Launch shape with the K dimension split across independent CTAs that add
// their FP32 partials through `part_bytes` of global workspace (gsplit_reduce):
// unlike a cluster split, any number of CTAs per SM and any split 1..8 can be
// used, so the weight stream can cover every SM.  One wave; the most weight
// bytes in flight (saturating at ~16 MB) wins, then the grid closest to two
// CTAs per SM.  Returns the dynamic shared memory size, or 0 when nothing fits.
template <int FMT>
int choose_shape_gpart(DParams& p, int n_tiles, const DeviceInfo& di, size_t part_bytes)
{
    if (p.M > kDecodeMaxGpartTokens) return 0;
    constexpr int64_t kSaturateBytes = 16ll << 20;
    const int stage_bytes = p.stage_bytes;
    int best_split = 0, best_stages = 0, best_smem = 0;
    int64_t best_score = -1;
    for (int sp = 1; sp <= kDecodeMaxSplit && sp <= p.k_stages; ++sp) {
        if (sp > 1 && (size_t)sp * n_tiles * p.M * DBM * 4 > part_bytes) break;
        const int per_cta_stages = (p.k_stages + sp - 1) / sp;
        for (int st = std::min(12, per_cta_stages); st >= std::min(2, per_cta_stages); --st) {
            const int smem = pad_smem_for_tmem(st * stage_bytes + 256 + 1024, p.tmem_cols, di);
            if ((size_t)smem > di.max_smem_optin) continue;
            const int active = max_resident_ctas<FMT>(1, smem, di);
            const int ctas = n_tiles * sp;
            if (active <= 0 || ctas > active) continue;
            const int64_t score = std::min<int64_t>(kSaturateBytes, (int64_t)ctas * st * stage_bytes) * 4096 +
                                  std::min(ctas, 2 * di.num_sms);
            if (score > best_score) {
                best_score = score;
                best_split = sp;
                best_stages = st;
                best_smem = smem;
            }
        }
    }
    if (best_split == 0) return 0;
    p.split = best_split;
    p.stages = best_stages;
    p.gpart = 1;
    p.bar_offset = p.stages * stage_bytes;
    return best_smem;
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
    attr[0].val.clusterDim.x = p.gpart ? 1u : (unsigned)p.split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // let the kernel be scheduled while its predecessor on the stream drains
    // (it waits for that kernel before touching what it may have written)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, tw, tx, tsfw, tsfx, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// ==========================================================================
// Uniform-NVFP4 decode with the token quantization inside the kernel
// ==========================================================================
//
// The tokens of a decode step are few (M <= 128), so every CTA quantizes the
// slice of X its K range needs itself, straight into shared memory in the MMA
// operand layout, while its producer warp already streams the weight: no
// separate quantization launch, no global round trip of the codes.  The
// dynamic tensor scale needs the maximum over all of X: each CTA takes the
// maximum of its K slice, and the CTAs of a cluster (whose slices cover all
// of K) exchange their maxima through distributed shared memory, so every
// cluster obtains the same alpha_x = amax / 2688 without touching global
// memory.
//
// Warps: 0 weight producer (TMA), 1 TMEM owner and MMA issuer, 2-9
// quantizers (warps 2-5 then drain the accumulator).  Shared memory: the
// weight ring (per stage 16 KiB of codes + 2 KiB of scale atoms), then the
// resident token slice (per K stage MT x 128 bytes of codes with the 128-byte
// swizzle + 2 KiB of scale atoms).
constexpr int F_THREADS = 320;
constexpr int F_QTHREADS = F_THREADS - 64;
constexpr int F_RING = QW_CODES + Q_SF;   // 18 KiB
constexpr int F_SMALL = 2048;             // barriers, exchange slots, encode table

struct FParams {
    const uint16_t* x;            // BF16 tokens [M, K]
    const float* alpha_static;    // or nullptr: dynamic alpha_x
    const float* alpha_w;
    int M, N, K, MT;
    int k_stages, split, stages;
    int x_off, x_stage;           // resident token slice: offset, bytes per K stage
    int bar_offset;
    uint32_t tmem_cols, tmem_sf;
    uint16_t* y;
    WsControl* ctrl;
    // K split across independent CTAs (see DParams): every CTA then takes the
    // amax over all of X itself instead of exchanging slice maxima in a cluster
    int gpart;
    float* part;
    uint32_t* tile_ctr;
};

__global__ void __launch_bounds__(F_THREADS, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_sfw,
                        const FParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + p.bar_offset);
    uint64_t* empty_bar = full_bar + p.stages;
    uint64_t* acc_full = empty_bar + p.stages;
    uint64_t* x_ready = acc_full + 1;
    uint64_t* amax_bar = x_ready + 1;
    uint32_t* amax_slot = reinterpret_cast<uint32_t*>(amax_bar + 1);   // [8], one per cluster rank
    uint32_t* red_q = amax_slot + 8;                                   // [F_QTHREADS / 32]
    uint32_t* tmem_slot = red_q + F_QTHREADS / 32;
    volatile uint32_t* abort_flag = tmem_slot + 1;
    uint32_t* s_last = tmem_slot + 2;
    float* enc_tab = reinterpret_cast<float*>(smem + p.bar_offset + 1024);   // [128]
    uint8_t* xr = smem + p.x_off;
    float* red = reinterpret_cast<float*>(smem);   // [MT][128] split-K partials, after the MMAs

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool cluster = p.split > 1 && !p.gpart;
    const uint32_t rank = (p.split > 1) ? (p.gpart ? (uint32_t)(blockIdx.x % p.split) : cluster_rank()) : 0u;
    const int n_tile = blockIdx.x / p.split;
    const int ks_begin = (int)(((int64_t)p.k_stages * rank) / p.split);
    const int ks_end = (int)(((int64_t)p.k_stages * (rank + 1)) / p.split);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(x_ready, F_QTHREADS);
        mbar_init(amax_bar, (uint32_t)p.split);
        *abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&tmap_w);
        prefetch_tensormap(&tmap_sfw);
    }
    if (warp == 1) tmem_alloc(tmem_slot, p.tmem_cols);
    tc_fence_before();
    __syncthreads();
    if (cluster) cluster_sync_all();   // every peer's barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    float alpha_x = 1.0f;
    grid_dep_wait();   // the previous kernel of the stream may have written X, W or Y
    grid_dep_launch_dependents();

    if (warp == 0) {
        // weight producer: whole warp, one elected lane issues
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int last_stage = -1;
        uint32_t last_parity = 0;
        for (int ks = ks_begin; ks < ks_end; ++ks) {
            if (!warp_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (elect_one()) {
                uint8_t* sw = smem + stage * F_RING;
                mbar_arrive_expect_tx(&full_bar[stage], (uint32_t)F_RING);
                tma_load_2d(sw, &tmap_w, &full_bar[stage], ks * (QBK / 2), n_tile * DBM);
                tma_load_2d(sw + QW_CODES, &tmap_sfw, &full_bar[stage], 0, n_tile * (p.k_stages * 4) + ks * 4);
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
            if (last_stage >= 0) (void)mbar_wait(&full_bar[last_stage], last_parity);
        }
    } else if (warp == 1) {
        // MMA issuer: waits once for the quantized tokens, then consumes the ring
        const uint32_t idesc = idesc_nvfp4(DBM, p.MT);
        const uint32_t sfa_tmem = tmem_base + p.tmem_sf;
        const uint32_t sfb_tmem = sfa_tmem + 16;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = warp_wait(x_ready, 0, abort_flag), next_ready = false;
        if (ok) tc_fence_after();
        for (int ks = ks_begin; ks < ks_end && ok; ++ks) {
            if (!next_ready && !warp_wait(&full_bar[stage], phase, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                const int ns = (stage + 1 == p.stages) ? 0 : stage + 1;
                next_ready = warp_test(&full_bar[ns], ns == 0 ? (phase ^ 1u) : phase);
            }
            const uint8_t* xs = xr + (ks - ks_begin) * p.x_stage;
            const uint64_t w_d = sdesc_kmajor_sw128(smem_u32(smem + stage * F_RING));
            const uint64_t x_d = sdesc_kmajor_sw128(smem_u32(xs));
            const uint64_t sfw_d = sdesc_sf_block(smem_u32(smem + stage * F_RING + QW_CODES));
            const uint64_t sfx_d = sdesc_sf_block(smem_u32(xs + p.MT * (QBK / 2)));
            if (elect_one()) {
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    tmem_cp_32x128b_x4(sfa_tmem + 4 * kb, sfw_d + (uint64_t)((kb * 512) >> 4));
                    tmem_cp_32x128b_x4(sfb_tmem + 4 * kb, sfx_d + (uint64_t)((kb * 512) >> 4));
                    umma_nvfp4(tmem_base, w_d + (uint64_t)((32 * kb) >> 4), x_d + (uint64_t)((32 * kb) >> 4), idesc,
                               sfa_tmem + 4 * kb, sfb_tmem + 4 * kb, (ks > ks_begin || kb > 0) ? 1u : 0u);
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
        if (elect_one()) tc_commit(acc_full);   // also "every MMA issued has finished" before TMEM is freed
        __syncwarp();
    } else {
        // ---- token quantization of this CTA's K slice [k_lo, k_hi), all M tokens
        const int qt = threadIdx.x - 64;
        const int qw = qt >> 5;
        const int nks = ks_end - ks_begin;
        const int k_lo = ks_begin * QBK;
        const int k_hi = min(ks_end * QBK, p.K);
        // scale atoms start at zero: padding rows (m >= M) and blocks past K then
        // contribute nothing to the MMA
        for (int i = qt; i < nks * (Q_SF / 16); i += F_QTHREADS) {
            const int s = i / (Q_SF / 16), j = i - s * (Q_SF / 16);
            reinterpret_cast<uint4*>(xr + s * p.x_stage + p.MT * (QBK / 2))[j] = make_uint4(0u, 0u, 0u, 0u);
        }
        bool ok = true;
        if (p.alpha_static != nullptr) {
            alpha_x = __ldg(p.alpha_static);
        } else {
            // |x| maximum of the slice (NaN/Inf excluded and flagged, as the amax pass
            // does); without a cluster to exchange slice maxima, of all of X
            const int a_lo = cluster ? k_lo : 0, a_hi = cluster ? k_hi : p.K;
            const int vpr = (a_hi - a_lo) / 8;
            uint32_t mx = 0, bad = 0;
            for (int v = qt; v < p.M * vpr; v += F_QTHREADS) {
                const int m = v / vpr, c = v - m * vpr;
                const uint4 q = __ldg(reinterpret_cast<const uint4*>(p.x + (int64_t)m * p.K + a_lo) + c);
                amax_accum(q.x, mx, bad);
                amax_accum(q.y, mx, bad);
                amax_accum(q.z, mx, bad);
                amax_accum(q.w, mx, bad);
            }
            uint32_t b = max(mx & 0xFFFFu, mx >> 16) | (bad ? 0x80000000u : 0u);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) b = fold_max_flag(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
            if (lane == 0) red_q[qw] = b;
            named_barrier_sync(1, F_QTHREADS);
            b = 0;
            for (int w = 0; w < F_QTHREADS / 32; ++w) b = fold_max_flag(b, red_q[w]);
            if (cluster) {
                // every rank's slice maximum into every rank's slot; the slots of all
                // ranks together cover K, so their fold is the maximum over all of X
                if (qt == 0) {
                    for (int q = 0; q < p.split; ++q) {
                        st_cluster_u32(map_to_cta(smem_u32(&amax_slot[rank]), (uint32_t)q), b);
                        mbar_arrive_cluster(map_to_cta(smem_u32(amax_bar), (uint32_t)q));
                    }
                }
                ok = mbar_wait_cluster(amax_bar, 0);
                b = 0;
                for (int q = 0; q < p.split; ++q) b = fold_max_flag(b, amax_slot[q]);
            }
            const float amax = __uint_as_float((b & 0x7FFFu) << 16);
            alpha_x = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
            if ((b & 0x80000000u) && qt == 0 && n_tile == 0 && rank == 0) post_error(p.ctrl, kErrNonFinite);
        }
        if (!ok) {
            if (qt == 0) post_error(p.ctrl, kErrTimeout);
            *abort_flag = 1;
        }
        const QuantConsts qc = quant_consts(alpha_x);
        if (qt < 128) {
            const float d = __fmul_rn(alpha_x, e4m3_to_float((uint32_t)qt));
            enc_tab[qt] = (d == 0.0f) ? 0.0f : __frcp_rn(d);
        }
        named_barrier_sync(1, F_QTHREADS);
        // Eq. 3 / Eq. 2 per 16-element block, written in the MMA operand layout:
        // codes row m of stage sl at (m/8)*1024 + (m%8)*128 + 16*(chunk ^ m%8),
        // scale (m, block kb) at the atom offset of the scale layout
        const int nb = (k_hi - k_lo) / 16;
        for (int b = qt; b < p.M * nb; b += F_QTHREADS) {
            const int m = b / nb, kb = b - m * nb;
            const uint4* src = reinterpret_cast<const uint4*>(p.x + (int64_t)m * p.K + k_lo + kb * 16);
            const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
            const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            uint32_t c0, c1;
            const uint32_t sc = quant_block16(w, qc, enc_tab, c0, c1);
            const int kbs = kb & 15;
            uint8_t* tile = xr + (kb >> 4) * p.x_stage;
            *reinterpret_cast<uint2*>(tile + (m >> 3) * 1024 + (m & 7) * 128 + ((((kbs >> 1) ^ (m & 7))) << 4) +
                                      (kbs & 1) * 8) = make_uint2(c0, c1);
            tile[p.MT * (QBK / 2) + (kbs >> 2) * 512 + (m & 31) * 16 + (m >> 5) * 4 + (kbs & 3)] = (uint8_t)sc;
        }
        fence_proxy_async_smem();   // the generic-proxy writes above are read by the tensor cores
        mbar_arrive(x_ready);

        if (warp < 6) {
            // ---- epilogue: warp w drains TMEM lane group w % 4
            const int lg = warp & 3;
            const int row = 32 * lg + lane;
            const int64_t n = (int64_t)n_tile * DBM + row;
            const float out_scale = __fmul_rn(__ldg(p.alpha_w), alpha_x);
            const bool have = mbar_wait(acc_full, 0) && !*abort_flag;
            if (!have && lane == 0) post_error(p.ctrl, kErrTimeout);
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(32 * lg) << 16);
            for (int c = 0; c < p.MT / 16; ++c) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(t_row + 16 * c, r);
                tmem_wait_ld(r);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int m = 16 * c + j;
                    const float v = have ? __uint_as_float(r[j]) : 0.0f;
                    if (p.split > 1 && p.gpart) {
                        if (m < p.M) p.part[(((int64_t)n_tile * p.split + rank) * p.M + m) * DBM + row] = v;
                    } else if (p.split > 1) {
                        red[m * DBM + row] = v;
                    } else if (m < p.M && n < p.N) {
                        p.y[(int64_t)m * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(v, out_scale)));
                    }
                }
            }
            if (p.split > 1 && p.gpart)
                gsplit_reduce(p.part, p.tile_ctr, s_last, n_tile, p.split, p.M, p.N, row,
                              warp == 2 && lane == 0, out_scale, p.y);
        }
    }

    if (cluster) {
        // every CTA of the cluster holds its partial tile; CTA `rank` sums tokens
        // m = rank, rank + split, ... over the ranks in rank order
        cluster_sync_all();
        if (warp >= 2 && warp < 6) {
            const int row = 32 * (warp & 3) + lane;
            const int64_t n = (int64_t)n_tile * DBM + row;
            const float out_scale = __fmul_rn(__ldg(p.alpha_w), alpha_x);
            for (int m = (int)rank; m < p.M; m += p.split) {
                float acc = 0.0f;
                const uint32_t laddr = smem_u32(&red[m * DBM + row]);
                for (int q = 0; q < p.split; ++q) acc += ld_dsmem_f32(laddr, (uint32_t)q);
                if (n < p.N) p.y[(int64_t)m * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(acc, out_scale)));
            }
        }
        cluster_sync_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

// Resident CTAs of decode_fused_kernel in clusters of `cluster` with `smem` bytes.
int fused_resident_ctas(int cluster, int smem, const DeviceInfo& di)
{
    static std::mutex mu;
    static std::map<std::tuple<int, int, int>, int> cache;
    const auto key = std::make_tuple(di.device, cluster, smem);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int ctas = 0;
    if (cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
        // nothing fits
    } else if (cluster == 1) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_fused_kernel, F_THREADS, smem) == cudaSuccess)
            ctas = per_sm * di.num_sms;
    } else {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)(cluster * di.num_sms), 1, 1);
        cfg.blockDim = dim3(F_THREADS, 1, 1);
        cfg.dynamicSmemBytes = (size_t)smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, decode_fused_kernel, &cfg) == cudaSuccess) ctas = clusters * cluster;
    }
    (void)cudaGetLastError();
    cache[key] = ctas;
    return ctas;
}

// BF16 decode of a single token on the CUDA cores: y[m, n] = bf16(sum_k
// W[n, k] x[m, k]) with FP32 fused multiply-adds.  For one token the
// tensor-core kernel spends its MMAs on padding (16 token columns) and each
// of its CTAs streams at the issue rate of its MMA loop; here the token sits
// in shared memory, and every warp streams whole weight rows with 16-byte
// loads (kGemvChunk per lane in flight, the whole 8 KiB row at K = 4096),
// multiplies them into two running sums per token, folds the sums over the
// warp and writes the row's outputs.  Warps take rows n, n + G, ... (G =
// warps in the grid), one wave of resident blocks.  Measured on the
// 12288 x 4096 weight: 22.5 vs 24.2 us per isolated call, 18.0 vs 20.3 us back
// to back; with two tokens the tensor-core kernel is the faster one (24.3 vs
// 26.4 us), so only single tokens come here.
constexpr int kGemvThreads = 256;
constexpr int kGemvChunk = 16;   // 16-byte vectors per lane per row chunk
constexpr int kGemvMaxTokens = 1;

template <int MT>
__global__ void __launch_bounds__(kGemvThreads) decode_gemv_kernel(const uint16_t* __restrict__ x,
                                                                   const uint16_t* __restrict__ w,
                                                                   uint16_t* __restrict__ y, int N, int K)
{
    extern __shared__ uint4 s_x[];   // MT token rows of K BF16 values
    grid_dep_wait();   // X may be the previous kernel's output
    grid_dep_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nv = K / 8;
    for (int i = threadIdx.x; i < MT * nv; i += kGemvThreads) s_x[i] = __ldg(reinterpret_cast<const uint4*>(x) + i);
    __syncthreads();
    const int64_t G = (int64_t)gridDim.x * (kGemvThreads / 32);
    for (int64_t n = (int64_t)blockIdx.x * (kGemvThreads / 32) + warp; n < N; n += G) {
        const uint4* wr = reinterpret_cast<const uint4*>(w + n * K);
        float acc[MT][2];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m][0] = acc[m][1] = 0.0f;
        for (int c0 = 0; c0 < nv; c0 += 32 * kGemvChunk) {
            uint4 v[kGemvChunk];
#pragma unroll
            for (int u = 0; u < kGemvChunk; ++u) {
                const int i = c0 + lane + 32 * u;
                v[u] = (i < nv) ? __ldcs(wr + i) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kGemvChunk; ++u) {
                const int i = c0 + lane + 32 * u;
                if (i < nv) {
                    const uint32_t wv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const uint4 xq = s_x[m * nv + i];
                        const uint32_t xv[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            acc[m][0] = __fmaf_rn(bf16_lo(wv[j]), bf16_lo(xv[j]), acc[m][0]);
                            acc[m][1] = __fmaf_rn(bf16_hi(wv[j]), bf16_hi(xv[j]), acc[m][1]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float a = __fadd_rn(acc[m][0], acc[m][1]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a = __fadd_rn(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
            if (lane == 0) y[(int64_t)m * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(a));
        }
    }
}

template <int MT>
cudaError_t launch_gemv(const void* x, const void* w, int64_t N, int64_t K, void* y, const DeviceInfo& di,
                        cudaStream_t s)
{
    const size_t smem = (size_t)MT * K * 2;
    auto kern = decode_gemv_kernel<MT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, smem) != cudaSuccess || per_sm < 1) {
        (void)cudaGetLastError();
        per_sm = 1;
    }
    int64_t blocks = (N + kGemvThreads / 32 - 1) / (kGemvThreads / 32);
    blocks = std::min<int64_t>(blocks, (int64_t)di.num_sms * per_sm);
    return launch_pdl(kern, dim3((unsigned)std::max<int64_t>(blocks, 1)), dim3(kGemvThreads), smem, s,
                      static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w), static_cast<uint16_t*>(y),
                      (int)N, (int)K);
}

}  // namespace

cudaError_t launch_decode_bf16(const void* x, int64_t M, const void* w, int64_t N, int64_t K, void* y,
                               WsControl* ctrl, const DecodeSplitWs& sw, const DeviceInfo& di, cudaStream_t s)
{
    // a single token: the CUDA-core kernel, if the token fits in shared memory
    if (M <= kGemvMaxTokens && (size_t)M * K * 2 <= di.max_smem_optin)
        return launch_gemv<kGemvMaxTokens>(x, w, N, K, y, di, s);
    DParams p{};
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.MT = (int)((M + 15) / 16 * 16);
    // two boxes (128 K elements) per stage once K has a few stages of them
    p.kbox = (K >= 8 * 2 * DBK) ? 2 : 1;
    p.k_stages = (int)((K + DBK * p.kbox - 1) / (DBK * p.kbox));
    p.tmem_cols = 32;
    while ((int)p.tmem_cols < p.MT) p.tmem_cols <<= 1;
    p.y = static_cast<uint16_t*>(y);
    p.ctrl = ctrl;
    p.stage_bytes = (W_STAGE + p.MT * DBK * 2) * p.kbox;
    const int n_tiles = (int)((N + DBM - 1) / DBM);
    p.part = sw.part;
    p.tile_ctr = sw.tile_ctr;
    int smem = (sw.part != nullptr) ? choose_shape_gpart<0>(p, n_tiles, di, sw.part_bytes) : 0;
    if (smem == 0) smem = choose_shape<0>(p, n_tiles, di);

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
                                int64_t K, void* y, WsControl* ctrl, const DecodeSplitWs& sw, const DeviceInfo& di,
                                cudaStream_t s)
{
    DParams p{};
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.MT = (int)((M + 31) / 32 * 32);   // MMA N: a multiple of 32, at most 128
    p.k_stages = (int)((K + QBK - 1) / QBK);
    p.kbox = 1;
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
    p.part = sw.part;
    p.tile_ctr = sw.tile_ctr;
    int smem = (sw.part != nullptr) ? choose_shape_gpart<1>(p, n_tiles, di, sw.part_bytes) : 0;
    if (smem == 0) smem = choose_shape<1>(p, n_tiles, di);

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

namespace mq {

cudaError_t launch_decode_nvfp4_fused(const void* x, int64_t M, const float* alpha_static, const uint8_t* w_codes,
                                      const uint8_t* w_scales, const float* alpha_w, int64_t N, int64_t K, void* y,
                                      WsControl* ctrl, const DecodeSplitWs& sw, const DeviceInfo& di, cudaStream_t s)
{
    FParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.alpha_static = alpha_static;
    p.alpha_w = alpha_w;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.MT = (int)((M + 31) / 32 * 32);   // MMA N: a multiple of 32, at most 128
    p.k_stages = (int)((K + QBK - 1) / QBK);
    uint32_t acc_cols = 32;
    while ((int)acc_cols < p.MT) acc_cols <<= 1;
    p.tmem_sf = acc_cols;
    p.tmem_cols = 32;
    while (p.tmem_cols < acc_cols + 32) p.tmem_cols <<= 1;
    p.x_stage = p.MT * (QBK / 2) + Q_SF;
    p.y = static_cast<uint16_t*>(y);
    p.ctrl = ctrl;
    const int n_tiles = (int)((N + DBM - 1) / DBM);

    // Launch shape: K split (cluster size) and ring depth.  Candidates must fit
    // the token slice and the ring in shared memory, run in one wave and leave
    // each CTA at most 32K token elements to quantize (every cluster quantizes
    // all tokens for its weight rows, so this work is repeated per 128 rows);
    // among them the most weight bytes in flight (saturating at ~16 MB) wins,
    // then the larger grid.
    //   With a partial workspace, the K split runs over independent CTAs (any
    // split 1..8, several CTAs per SM; each CTA takes the amax over all of X,
    // so only for at most 64K elements: beyond that every CTA re-reading all
    // tokens costs more than a cluster's exchange of slice maxima); otherwise
    // over a cluster (split a power of two).
    constexpr int64_t kSaturateBytes = 16ll << 20;
    int best_split = 0, best_st = 0, best_smem = 0, best_gpart = 0;
    int64_t best_score = -1;
    const bool can_gpart = sw.part != nullptr && M <= kDecodeMaxGpartTokens &&
                           (p.alpha_static != nullptr || M * K <= (int64_t)1 << 16);
    for (int sp = 1; sp <= 8 && sp <= p.k_stages; ++sp) {
        const bool gp = can_gpart && (sp == 1 || (size_t)sp * n_tiles * M * DBM * 4 <= sw.part_bytes);
        if (!gp && (sp & (sp - 1)) != 0) continue;   // a cluster split is a power of two
        const int nks = (p.k_stages + sp - 1) / sp;
        for (int st = std::min(8, nks); st >= std::min(2, nks); --st) {
            const int body = std::max(st * F_RING + nks * p.x_stage, p.MT * DBM * 4);
            int smem = (body + 1023) / 1024 * 1024 + F_SMALL + 1024;
            // TMEM: the CTAs that can share an SM must fit its 512 columns (an
            // allocation that cannot be served would wait for a CTA that may itself
            // wait on a cluster peer), so pad the shared memory to cap them
            const int tmem_cap = 512 / (int)p.tmem_cols;
            const int per_sm_min = (int)(di.smem_per_sm / (size_t)(tmem_cap + 1)) + 1;   // bytes incl. reserve
            smem = std::max<int>(smem, per_sm_min - (int)di.smem_reserved_per_cta);
            smem = (smem + 1023) / 1024 * 1024;
            if ((size_t)smem > di.max_smem_optin) continue;
            const int ctas = n_tiles * sp;
            const int active = fused_resident_ctas(gp ? 1 : sp, smem, di);
            if (active <= 0 || ctas > active) continue;
            if (M * (K / sp) > 32768) continue;
            const int64_t score = std::min<int64_t>(kSaturateBytes, (int64_t)ctas * st * F_RING) * 4096 +
                                  std::min(ctas, 2 * di.num_sms);
            if (score > best_score) {
                best_score = score;
                best_split = sp;
                best_st = st;
                best_smem = smem;
                best_gpart = gp ? 1 : 0;
            }
        }
    }
    if (best_split == 0) return cudaErrorNotSupported;   // the caller takes the two-kernel path
    p.split = best_split;
    p.stages = best_st;
    p.gpart = best_gpart;
    p.part = sw.part;
    p.tile_ctr = sw.tile_ctr;
    const int nks = (p.k_stages + p.split - 1) / p.split;
    p.x_off = p.stages * F_RING;
    const int body = std::max(p.x_off + nks * p.x_stage, p.MT * DBM * 4);
    p.bar_offset = (body + 1023) / 1024 * 1024;

    CUtensorMap tw, tsfw;
    if (!make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, (uint64_t)(K / 2), (uint64_t)N, (uint64_t)(K / 2),
                      QBK / 2, DBM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tsfw, CU_TENSOR_MAP_DATA_TYPE_UINT32, w_scales, 128,
                      (uint64_t)sf_rowblks(N) * (uint64_t)sf_atoms_per_rowblk(K), 512, 128, 4,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, best_smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(n_tiles * p.split), 1, 1);
    cfg.blockDim = dim3(F_THREADS, 1, 1);
    cfg.dynamicSmemBytes = (size_t)best_smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.gpart ? 1u : (unsigned)p.split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, decode_fused_kernel, tw, tsfw, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace mq
