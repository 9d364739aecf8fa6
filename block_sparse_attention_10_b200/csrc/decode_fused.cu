// decode_fused.cu — the whole MSA decode step (index -> pool -> select -> attend) in
// one persistent launch.
//
// Prior art: a single-launch "mono" decode path that replaces the many launches of a
// decode step ("vLLM turns MiniMax's day-zero promise into GPU-specific serving code",
// upstreambeat.ai, "What changed").  The arithmetic is that of the separate kernels —
// index_block.cuh (indexer + pooling), select_row.cuh (top-16, recent block forced),
// attend_quarter.cuh (exact attention) — only the scheduling differs.
//
// Design (B200):
//   * 2 CTAs x 8 warps per SM.  The W warps of the grid share one ordered work list;
//     warp w takes items w, w + W, w + 2W, ... (no atomics; the next item is always
//     known, so a warp's copies run ahead across item boundaries).  Items:
//       IDX (b, n0..n1)     score + pool a run of blocks of sequence b (HBM stream);
//       SEL (b, t)          top-16 of row (b, t) once every block of b is pooled;
//       ATT (b, t, kvh, a)  attention of the G query heads of KV head kvh over the
//                           row's selected blocks 2a, 2a+1 -> a partial (m, l, O) in
//                           the workspace; the warp that completes a (row, KV head)'s
//                           8th partial merges them, in slot order (deterministic).
//     At step k the list holds the IDX items of sequence k, then the SEL items of
//     sequence k - lag_s, then the ATT items of sequence k - lag_a, the lags being
//     about one round of W items each: the attention of early sequences (issue-bound)
//     runs while later sequences' keys stream in (HBM-bound), and a sequence's
//     selection and attention rarely wait for the items they depend on.
//   * Every item depends only on items earlier in the list.  All warps must be
//     resident for the waits to end: the grid is sized to the occupancy limit, and a
//     wait for another warp's result gives up after 2 s, setting a status bit and an
//     abort flag that ends every other wait at once (never a hang).
//   * Each warp streams all its operands through one private ring of 3 shared-memory
//     stages of 4.5 KB (an index-key stage and an attention quarter have the same
//     size): lane 0 issues the bulk copies (cp.async.bulk, no multicast) of the current
//     item and of the next one as soon as it is known, up to 2 stages ahead.
//   * Workspace: [counters][pooled scores][selection][partials]; the counters are
//     cleared by the host before every launch.
#include <algorithm>

#include "attend_quarter.cuh"
#include "index_block.cuh"
#include "select_row.cuh"

namespace msa {
namespace {

constexpr int kFWarps = 8;
constexpr int kFThreads = 32 * kFWarps;
constexpr int kFRing = 3;
constexpr int kFStage = kIdxStageBytes;
static_assert(kIdxStageBytes == kAttStageBytes, "index and attention stages share the ring");
constexpr int kItemStages = 8;  // stages per IDX item: 4 blocks at DI = 128, 8 at DI = 64
constexpr int kAttBlocksPerItem = 2;
constexpr int kAttItemsPerRow = kTopK / kAttBlocksPerItem;  // partials per (row, KV head)
constexpr int kPartFloats = 64 * 8 * 2 + 16;                // O [64 dim pairs][8 heads][2], m[8], l[8]
constexpr int kMaxB = 4096;

// counter words
constexpr int kCtrAbort = 0, kCtrHeader = 4;

enum : int { kEnd = 0, kIdx = 1, kSel = 2, kAtt = 3 };

struct FArgs {
    uint32_t* ctr;       // [kCtrHeader + B + B*Tq + B*Tq*Hkv]
    float* bscores;      // [B][Tq][nbmax]
    int32_t* sel;        // [B][Tq][16]
    float* part;         // [B*Tq*Hkv][kAttItemsPerRow][kPartFloats]
    float* out;
    float* lse;
    int lag_s, lag_a;    // list steps from IDX(b) to SEL(b) and to ATT(b)
};

// One work item as every lane of the warp sees it.
struct FItem {
    int type;
    int b, t, kvh, a;  // IDX: blocks [a, t) of sequence b; SEL: row (b, t); ATT: see above
    int nst;           // stages in the ring (-1: ATT whose selection is not read yet)
    int blk0, blk1;    // ATT: the two selected blocks (-1: none)
    int nk0, nk1;      // ATT: their visible keys
};
static_assert(kAttBlocksPerItem == 2, "FItem holds two blocks per ATT item");

constexpr size_t f_smem_bytes(int B) {
    return (size_t)kFWarps * kFRing * (kFStage + sizeof(uint64_t)) + (size_t)(2 * B + 2) * sizeof(int);
}

// List position of step k's first item: the IDX, SEL and ATT items of all earlier steps.
__device__ __forceinline__ int64_t f_pos(int64_t k, const int* pre, int B, int Tq, int64_t att_per_seq, int lag_s,
                                         int lag_a) {
    auto clampB = [&](int64_t x) { return x < 0 ? 0 : (x > B ? (int64_t)B : x); };
    return pre[k < B ? k : B] + (int64_t)Tq * clampB(k - lag_s) + att_per_seq * clampB(k - lag_a);
}

template <int DI, int HI, int NT>
__global__ void __launch_bounds__(kFThreads, 2) decode_fused_kernel(const Problem p, const FArgs fa) {
    constexpr int R = kFRing;
    constexpr int KPS = idx_stage_keys<DI>();
    constexpr int SPB = kBlock / KPS;           // stages per full block
    constexpr int CB = kItemStages / SPB;       // blocks per IDX item

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kFWarps * R * kFStage);
    int* pre = reinterpret_cast<int*>(bars + kFWarps * R);  // [B + 1] IDX items before sequence b
    int* lens = pre + (p.B + 1);                            // [B] clamped lengths

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int B = p.B, Tq = p.Tq, Hkv = p.Hkv;
    const int G = p.Hq / p.Hkv;
    uint8_t* my_stages = smem + warp * R * kFStage;
    uint64_t* my_bars = bars + warp * R;
    uint32_t* idx_done = fa.ctr + kCtrHeader;       // [B] blocks pooled
    uint32_t* sel_ready = idx_done + B;             // [B*Tq]
    uint32_t* att_done = sel_ready + (int64_t)B * Tq;  // [B*Tq*Hkv] partials written
    uint32_t* abort_flag = fa.ctr + kCtrAbort;

    if (lane == 0) {
        for (int s = 0; s < R; ++s) mbar_init(&my_bars[s], 1);
        fence_mbar_init();
    }
    pdl_wait();
    if (warp == 0) {
        int carry = 0;
        if (lane == 0) pre[0] = 0;
        for (int b0 = 0; b0 < B; b0 += 32) {
            const int b = b0 + lane;
            int ni = 0;
            if (b < B) {
                const int64_t L = clamp_len(p.seq_lens[b], Tq, p.lmax, blockIdx.x == 0 ? p.status : nullptr);
                lens[b] = (int)L;
                ni = (int)(((L + kBlock - 1) / kBlock + CB - 1) / CB);
            }
            int x = ni;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (b < B) pre[b + 1] = carry + x;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
    }
    __syncthreads();
    pdl_launch_dependents();

    const int64_t att_per_seq = (int64_t)Tq * Hkv * kAttItemsPerRow;
    const int lag_s = fa.lag_s, lag_a = fa.lag_a;
    const int64_t ksteps = (int64_t)B + lag_a;
    const int64_t total = f_pos(ksteps, pre, B, Tq, att_per_seq, lag_s, lag_a);
    const float sc_log2 = p.softmax_scale * p.k.s_t * kLog2e;

    auto aborted = [&]() -> bool { return *reinterpret_cast<volatile uint32_t*>(abort_flag) != 0u; };
    auto fail = [&](uint32_t where) {
        if (lane == 0) {
            set_status(p.status, MSA_STATUS_TIMEOUT | where);
            atomicExch(abort_flag, 1u);
        }
    };
    // lane 0 polls until *ctr >= target (acquire), the abort flag, or the time limit
    auto wait_geq = [&](const uint32_t* ctr, uint32_t target) -> bool {
        int ok = 1;
        if (lane == 0 && ld_acquire_u32(ctr) < target) {
            const uint64_t t0 = globaltimer_ns();
            for (;;) {
                __nanosleep(200);
                if (ld_acquire_u32(ctr) >= target) break;
                if (aborted()) {
                    ok = 0;
                    break;
                }
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    ok = 0;
                    set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_DECODE_WAIT);
                    atomicExch(abort_flag, 1u);
                    break;
                }
            }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __threadfence();
        return ok != 0;
    };

    auto decode_ticket = [&](int64_t x) -> FItem {
        FItem it;
        it.type = kEnd;
        it.nst = 0;
        if (x >= total) return it;
        // last step k with f_pos(k) <= x
        int64_t lo = 0, hi = ksteps - 1;
        while (lo < hi) {
            const int64_t mid = (lo + hi + 1) >> 1;
            if (f_pos(mid, pre, B, Tq, att_per_seq, lag_s, lag_a) <= x) lo = mid;
            else hi = mid - 1;
        }
        const int64_t k = lo;
        int64_t o = x - f_pos(k, pre, B, Tq, att_per_seq, lag_s, lag_a);
        if (k < B) {
            const int64_t ni = pre[k + 1] - pre[k];
            if (o < ni) {
                const int b = (int)k;
                const int64_t L = lens[b];
                const int nb = (int)((L + kBlock - 1) / kBlock);
                it.type = kIdx;
                it.b = b;
                it.a = (int)o * CB;
                it.t = min(nb, it.a + CB);
                it.nst = (it.t - it.a - 1) * SPB + idx_block_stages<DI>(it.t - 1, L);
                return it;
            }
            o -= ni;
        }
        if (k - lag_s >= 0 && k - lag_s < B) {
            if (o < Tq) {
                it.type = kSel;
                it.b = (int)(k - lag_s);
                it.t = (int)o;
                return it;
            }
            o -= Tq;
        }
        if (k - lag_a < 0 || k - lag_a >= B) return it;  // unreachable: the steps' sizes add up to total
        it.type = kAtt;
        it.b = (int)(k - lag_a);
        it.t = (int)(o / ((int64_t)Hkv * kAttItemsPerRow));
        it.kvh = (int)((o / kAttItemsPerRow) % Hkv);
        it.a = (int)(o % kAttItemsPerRow);
        it.nst = -1;
        return it;
    };
    // reads an ATT item's selected blocks if its row is selected (no waiting)
    auto att_resolve = [&](FItem& it) -> bool {
        const int64_t row = (int64_t)it.b * Tq + it.t;
        uint32_t ready = lane == 0 ? ld_acquire_u32(sel_ready + row) : 0u;
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (ready == 0u) return false;
        __threadfence();
        const int64_t pos = (int64_t)lens[it.b] - Tq + it.t;
        int blk[2], nk[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            blk[j] = __ldcg(fa.sel + row * kTopK + it.a * kAttBlocksPerItem + j);
            if (blk[j] > pos / kBlock) {  // not a visible block
                if (lane == 0) set_status(p.status, MSA_STATUS_SELECT);
                blk[j] = -1;
            }
            nk[j] = blk[j] >= 0 ? (int)min64(kBlock, pos + 1 - (int64_t)blk[j] * kBlock) : 0;
        }
        it.blk0 = blk[0];
        it.blk1 = blk[1];
        it.nk0 = nk[0];
        it.nk1 = nk[1];
        it.nst = (nk[0] + kAttQuarter - 1) / kAttQuarter + (nk[1] + kAttQuarter - 1) / kAttQuarter;
        return true;
    };

    // ---- the warp's ring: issue side walks (item, stage) over cur then nxt
    const int64_t W = (int64_t)gridDim.x * kFWarps;
    int64_t ticket = (int64_t)blockIdx.x * kFWarps + warp;  // list position of cur
    FItem cur, nxt;
    bool nxt_valid = false;
    bool nxt_tried = false;  // one non-waiting look at an ATT nxt's selection per item
    int iw = 0, isi = 0;     // issue position: item (0 cur, 1 nxt), stage in it
    uint32_t slot = 0, slot_issued = 0;
    auto issue_stage = [&](const FItem& it, int si) {
        const int s = (int)(slot_issued % R);
        uint8_t* st = my_stages + s * kFStage;
        if (lane == 0) {
            if (it.type == kIdx) {
                const int n = it.a + si / SPB, sub = si % SPB;
                const int valid = (int)min64(kBlock, (int64_t)lens[it.b] - (int64_t)n * kBlock) - sub * KPS;
                const int rows = (min(valid, KPS) + 15) & ~15;
                const int64_t row0 = (int64_t)it.b * p.lmax + (int64_t)n * kBlock + sub * KPS;
                const uint32_t db = (uint32_t)(rows * (DI / 2)), sb = (uint32_t)(rows * (DI / 16));
                mbar_arrive_expect_tx(&my_bars[s], db + sb);
                bulk_g2s(st, p.ik.data + row0 * (DI / 2), db, &my_bars[s]);
                bulk_g2s(st + kIdxStageData, p.ik.scale + row0 * (DI / 16), sb, &my_bars[s]);
            } else {
                const int nq0 = (it.nk0 + kAttQuarter - 1) / kAttQuarter;
                const bool second = si >= nq0;
                const int qq = second ? si - nq0 : si;
                const int nk = second ? it.nk1 : it.nk0, blk = second ? it.blk1 : it.blk0;
                const int rows = (min(kAttQuarter, nk - qq * kAttQuarter) + 15) & ~15;
                const int64_t vec = ((int64_t)it.b * Hkv + it.kvh) * p.lmax + (int64_t)blk * kBlock + qq * kAttQuarter;
                att_issue_quarter(p, st, vec, rows, &my_bars[s]);
            }
        }
        ++slot_issued;
    };
    auto fetch_nxt = [&]() {
        if (!nxt_valid) {
            nxt = decode_ticket(ticket + W);
            nxt_valid = true;
        }
    };
    auto issue_upto = [&](uint32_t limit) {
        while (slot_issued < limit) {
            if (iw == 0) {
                if (cur.nst < 0 && !att_resolve(cur)) break;
                if (isi < cur.nst) {
                    issue_stage(cur, isi++);
                    continue;
                }
                if (cur.type == kEnd) break;
                fetch_nxt();
                iw = 1;
                isi = 0;
            } else {
                if (nxt.type == kEnd) break;
                if (nxt.nst < 0) {
                    if (nxt_tried) break;
                    nxt_tried = true;
                    if (!att_resolve(nxt)) break;
                }
                if (isi < nxt.nst) {
                    issue_stage(nxt, isi++);
                    continue;
                }
                break;
            }
        }
    };
    // the next stage of the warp's stream (in order), or nullptr after a timeout
    auto acquire = [&]() -> const uint8_t* {
        issue_upto(slot + R);
        const int s = (int)(slot % R);
        if (!mbar_wait(&my_bars[s], (slot / R) & 1u)) {
            fail(MSA_STATUS_AT_DECODE_STAGE);
            return nullptr;
        }
        ++slot;
        return my_stages + s * kFStage;
    };

    cur = decode_ticket(ticket);
    bool ok = true;
    while (cur.type != kEnd && ok) {
        if (cur.type == kIdx) {
            // ---------------------------------------------------------------- index
            IdxQuery<DI, NT> q;
            idx_load_query<DI, HI, NT>(p, cur.b, g, c, q);
            const int64_t L = lens[cur.b];
            for (int n = cur.a; n < cur.t && ok; ++n)
                ok = idx_block<DI, HI, NT>(p, cur.b, n, L, q, acquire, fa.bscores, nullptr, g, c);
            if (!ok) break;
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(idx_done + cur.b, (uint32_t)(cur.t - cur.a));
        } else if (cur.type == kSel) {
            // ---------------------------------------------------------------- select
            const int64_t L = lens[cur.b];
            const int nb = (int)((L + kBlock - 1) / kBlock);
            issue_upto(slot + R);  // prefetch the next item's stages while waiting
            if (!wait_geq(idx_done + cur.b, (uint32_t)nb)) break;
            const int64_t row = (int64_t)cur.b * Tq + cur.t;
            const int64_t pos = L - Tq + cur.t;
            const int64_t nvis = pos / kBlock + 1;
            if (nvis <= 512) {
                select_row_warp<16, true>(fa.bscores + row * p.nbmax, nvis, nvis - 1, lane, fa.sel + row * kTopK);
            } else {
                const int id = select_row_warp_long<16, true>(fa.bscores + row * p.nbmax, nvis, nvis - 1, lane);
                if (lane < kTopK) fa.sel[row * kTopK + lane] = id;
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_u32(sel_ready + row, 1u);
        } else {
            // ---------------------------------------------------------------- attend
            const int64_t row = (int64_t)cur.b * Tq + cur.t;
            if (cur.nst < 0) {
                if (!wait_geq(sel_ready + row, 1u)) break;
                att_resolve(cur);
            }
            uint32_t qf[1][8][2];
            att_load_q(p, row, cur.kvh, G, g, c, qf);
            AttAcc acc;
            att_init(acc);
            // stage si: quarter si of the first block, then the quarters of the second
            const int nq0 = (cur.nk0 + kAttQuarter - 1) / kAttQuarter;
            for (int si = 0; si < cur.nst; ++si) {
                const uint8_t* st = acquire();
                if (st == nullptr) {
                    ok = false;
                    break;
                }
                const int left = si < nq0 ? cur.nk0 - si * kAttQuarter : cur.nk1 - (si - nq0) * kAttQuarter;
                att_quarter(st, min(kAttQuarter, left), si == 0, qf, sc_log2, g, c, acc);
                __syncwarp();  // every lane is done with the stage before it is refilled
            }
            if (!ok) break;
            att_reduce_l(acc);
            const int64_t rk = row * Hkv + cur.kvh;
            float* part = fa.part + (rk * kAttItemsPerRow + cur.a) * kPartFloats;
            att_store_o(part, g, c, acc);
            if (g == 0) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    part[1024 + 2 * c + e] = acc.m2[e];
                    part[1032 + 2 * c + e] = acc.l2[e];
                }
            }
            __threadfence();
            __syncwarp();
            uint32_t prev = 0;
            if (lane == 0) prev = atomicAdd(att_done + rk, 1u);
            prev = __shfl_sync(0xffffffffu, prev, 0);
            if (prev == kAttItemsPerRow - 1) {
                // last partial of (row, kvh): merge all of them in slot order
                __threadfence();
                const float* base = fa.part + rk * kAttItemsPerRow * kPartFloats;
                const int h0 = 2 * (lane & 3);
                float M[2] = {-INFINITY, -INFINITY};
                float mw[kAttItemsPerRow][2];
#pragma unroll
                for (int i = 0; i < kAttItemsPerRow; ++i) {
                    const float2 m = __ldcg(reinterpret_cast<const float2*>(base + i * kPartFloats + 1024 + h0));
                    mw[i][0] = m.x;
                    mw[i][1] = m.y;
                    M[0] = fmaxf(M[0], m.x);
                    M[1] = fmaxf(M[1], m.y);
                }
                float Lt[2] = {0.0f, 0.0f};
#pragma unroll
                for (int i = 0; i < kAttItemsPerRow; ++i) {
                    const float2 l = __ldcg(reinterpret_cast<const float2*>(base + i * kPartFloats + 1032 + h0));
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        mw[i][e] = mw[i][e] == -INFINITY ? 0.0f : exp2f(mw[i][e] - M[e]);
                        Lt[e] += mw[i][e] * (e == 0 ? l.x : l.y);
                    }
                }
                float4 o4[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) o4[k] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
                for (int i = 0; i < kAttItemsPerRow; ++i) {
                    const float4* src = reinterpret_cast<const float4*>(base + i * kPartFloats);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float4 v = __ldcg(src + lane + 32 * k);  // dim pair (lane >> 2) + 8k, heads h0, h0+1
                        o4[k].x += mw[i][0] * v.x;
                        o4[k].y += mw[i][0] * v.y;
                        o4[k].z += mw[i][1] * v.z;
                        o4[k].w += mw[i][1] * v.w;
                    }
                }
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int h = h0 + e;
                    if (h < G) {
                        const float inv = Lt[e] > 0.0f ? p.v.s_t / Lt[e] : 0.0f;
                        const int64_t orow = (row * p.Hq + (int64_t)cur.kvh * G + h) * kAttD;
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const int pi = (lane >> 2) + 8 * k;
                            if (e == 0) store_out2(p, fa.out, orow + 2 * pi, o4[k].x * inv, o4[k].y * inv);
                            else store_out2(p, fa.out, orow + 2 * pi, o4[k].z * inv, o4[k].w * inv);
                        }
                        if (fa.lse != nullptr && lane < 4)
                            fa.lse[row * p.Hq + (int64_t)cur.kvh * G + h] =
                                Lt[e] > 0.0f ? (M[e] + log2f(Lt[e])) * kLn2 : -INFINITY;
                    }
                }
            }
        }
        // next item
        fetch_nxt();
        cur = nxt;
        ticket += W;
        nxt_valid = false;
        nxt_tried = false;
        if (iw == 1) iw = 0;
        else isi = 0;
    }
    // never leave with copies in flight into this warp's stages
    for (uint32_t j = slot; j < slot_issued; ++j)
        if (!mbar_wait(&my_bars[j % R], (j / R) & 1u)) {
            if (lane == 0) set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_DECODE_STAGE);
            break;
        }
}

template <int DI, int HI, int NT>
int launch_t(const Problem& p, const FArgs& fa, bool pdl, cudaStream_t st) {
    auto kern = decode_fused_kernel<DI, HI, NT>;
    const size_t smem = f_smem_bytes(p.B);
    static int configured_dev = -1;
    const DeviceInfo& di = device_info();
    if (configured_dev != di.device) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)f_smem_bytes(kMaxB)) !=
            cudaSuccess)
            return MSA_ECUDA;
        configured_dev = di.device;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFThreads, smem) != cudaSuccess || per_sm < 1)
        return MSA_ECUDA;
    const int grid = min(per_sm, 2) * di.num_sms;
    // lags of about one round (W items) each: a sequence's SEL item comes about one
    // round after its last IDX item, its ATT items one more round later
    // (items per step estimated from lmax: the lengths are on the device)
    FArgs f = fa;
    const int64_t W = (int64_t)grid * kFWarps;
    constexpr int CB = kItemStages / (kBlock / idx_stage_keys<DI>());
    const int64_t per_step = (p.nbmax + CB - 1) / CB + p.Tq + (int64_t)p.Tq * p.Hkv * kAttItemsPerRow;
    const int64_t lag = (W + per_step - 1) / per_step;
    f.lag_s = (int)std::min<int64_t>(p.B, std::max<int64_t>(1, lag));
    f.lag_a = (int)std::min<int64_t>((int64_t)p.B + f.lag_s, f.lag_s + std::max<int64_t>(1, lag));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, p, f) != cudaSuccess) return MSA_ECUDA;
    return MSA_OK;
}

template <int DI, int HI>
int launch_nt(const Problem& p, const FArgs& fa, bool pdl, cudaStream_t st) {
    const int nq = p.Tq * HI;
    if (nq <= 8) return launch_t<DI, HI, 1>(p, fa, pdl, st);
    if (nq <= 16) return launch_t<DI, HI, 2>(p, fa, pdl, st);
    return MSA_EUNSUPPORTED;
}

template <int DI>
int launch_hi(const Problem& p, const FArgs& fa, bool pdl, cudaStream_t st) {
    switch (p.HI) {
        case 1: return launch_nt<DI, 1>(p, fa, pdl, st);
        case 2: return launch_nt<DI, 2>(p, fa, pdl, st);
        case 4: return launch_nt<DI, 4>(p, fa, pdl, st);
        case 8: return launch_nt<DI, 8>(p, fa, pdl, st);
        default: return MSA_EUNSUPPORTED;
    }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

FusedLayout fused_layout(const Problem& p) {
    FusedLayout l;
    const size_t rows = (size_t)p.B * p.Tq;
    l.ctr_bytes = align256((kCtrHeader + (size_t)p.B + rows + rows * p.Hkv) * sizeof(uint32_t));
    l.bscores = l.ctr_bytes;
    l.sel = l.bscores + align256(rows * (size_t)p.nbmax * sizeof(float));
    l.part = l.sel + align256(rows * kTopK * sizeof(int32_t));
    l.total = l.part + align256(rows * p.Hkv * (size_t)kAttItemsPerRow * kPartFloats * sizeof(float));
    return l;
}

bool fused_supported(const Problem& p) {
    return p.B <= kMaxB && (int64_t)p.Tq * p.HI <= 16 && (p.DI == 64 || p.DI == 128) && p.D == kAttD &&
           p.block_table == nullptr;
}

int launch_decode_fused(const Problem& p, void* ws, float* out, float* lse, int32_t* sel_out, bool pdl,
                        cudaStream_t st) {
    if (!fused_supported(p)) return MSA_EUNSUPPORTED;
    const FusedLayout l = fused_layout(p);
    uint8_t* w = static_cast<uint8_t*>(ws);
    FArgs fa;
    fa.ctr = reinterpret_cast<uint32_t*>(w);
    fa.bscores = reinterpret_cast<float*>(w + l.bscores);
    fa.sel = sel_out != nullptr ? sel_out : reinterpret_cast<int32_t*>(w + l.sel);
    fa.part = reinterpret_cast<float*>(w + l.part);
    fa.out = out;
    fa.lse = lse;
    if (cudaMemsetAsync(fa.ctr, 0, l.ctr_bytes, st) != cudaSuccess) return MSA_ECUDA;
    if (p.DI == 128) return launch_hi<128>(p, fa, pdl, st);
    return launch_hi<64>(p, fa, pdl, st);
}

}  // namespace msa
