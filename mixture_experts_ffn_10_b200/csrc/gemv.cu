// gemv.cu -- the forward of a handful of tokens (T <= kGemvMaxTokens, bf16 weights)
// in one cooperative launch: routing, gate_up with its activation, down with bias
// and routing weight, and the combine.  With so few tokens the layer is a stream of
// the chosen experts' weights (each read once), so the kernel is built around that
// stream: every warp pulls its own 8 KiB weight tiles with TMA and multiplies each
// by the tokens' rows with warp-level mma.sync (m16n8k16: 16 weight rows x 16 K
// against 8 columns, the token slots of the tile's expert), which costs a handful of
// instructions per tile where CUDA-core dot products cost one per weight.
//
// Definitions (the same as the multi-launch path; "Struct MoeSpec" act, weigh_inputs;
// graph-op page "MoE" gate/up stacks and fusion_size; "ClikaRT::nn::QMoEWoQ" forward):
//   h[(t,j), f] = act(wi g + bg) (wi u + bu), g/u = x_t . gate/up row f of expert e_tj,
//                 wi = w_tj with weigh-inputs, else 1;  plain: act(wi v + b)
//   Y[(t,j), n] = bf16((h . down row n + b_n) * w_tj)   (w = 1 with weigh-inputs and
//                 for the shared expert)
//   y[t, n]     = sum_j Y[(t,j), n] + gate_t Y_shared[t, n] + shared_output[t, n],
//                 in fp32 in this order, rounded once
// h and Y are rounded to bf16 as in the tensor-core path.  Each warp's instruction
// sequence is fixed by the shapes, so results repeat bitwise from run to run.
//
// Work: gate_up jobs (8 gated features = their 8 gate and 8 up rows, or 16 plain
// features) and down units (16 output features of one chosen expert), each split in
// stages of kGemvKS along K; job / unit i goes to CTA i mod G and, inside it, to warp
// (i div G) mod W, down units continuing the rotation where the jobs stop.  Each warp
// keeps kGemvSlotsPerWarp stages in flight.  Between the phases every CTA publishes
// its h features (one release increment) and waits for all CTAs; the slots already
// hold the first down stages meanwhile.  A down unit writes its Y rows; the last of
// the units of a 16-feature row block (a per-block counter) combines that block.
#include "epilogue.cuh"
#include "gemv.cuh"
#include "route.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int SPW = kGemvSlotsPerWarp;
constexpr int kKB = kGemvKB;
constexpr int kKS = kGemvKS;
constexpr int kSlot = kGemvSlotBytes;
constexpr int kRB = kGemvRowBlock;
constexpr int kAcc = 4;  // independent accumulator sets per warp

__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

// Bounded wait for the phase of `bar` with the given parity that suspends the warp
// (suspend-time hint) instead of spinning, so that waiting warps leave the issue slots
// to the warps that have data.  Gives up like mbar_wait: on *abort, or after
// kTimeoutNs (then it sets *abort and records MOE_ERR_TIMEOUT).
__device__ __forceinline__ bool wait_tile(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
  constexpr uint32_t kHintNs = 20000;
  const uint64_t t0 = global_timer();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kHintNs)
        : "memory");
    if (ok) return true;
    if (*abort) return false;
    if (global_timer() - t0 > kTimeoutNs) {
      *abort = 1;
      set_status(status, MOE_ERR_TIMEOUT);
      return false;
    }
  }
}

// D += A B for one 16 x 16 (rows x K) bf16 tile A and 16 x 8 (K x columns) bf16 B.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Position in the expert list of a monotone walk over gate_up jobs: entry u owns jobs
// u0 .. u0 + (its features / fj) - 1.
struct JobCursor {
  int u = 0, u0 = 0;
  __device__ __forceinline__ void seek(const GemvMeta& m, const GemvArgs& a, int fj, int job) {
    while (job >= u0 + (m.e[u] < 0 ? a.Fs : a.F) / fj) u0 += (m.e[u++] < 0 ? a.Fs : a.F) / fj;
  }
};

template <int EPL>
__global__ void __launch_bounds__(kGemvMaxWarps * 32, 1)
    gemv_ffn_kernel(const __grid_constant__ CUtensorMap tm_gu, const __grid_constant__ CUtensorMap tm_gu2,
                    const __grid_constant__ CUtensorMap tm_sgu, const __grid_constant__ CUtensorMap tm_dn,
                    const __grid_constant__ CUtensorMap tm_sdn, const __grid_constant__ GemvArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kGemvMaxWarps * SPW];
  __shared__ GemvMeta m;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;  // mma fragment coordinates
  const int NW = a.warps;
  const int T = a.T, k = a.k, d = a.d, R = a.R;
  uint8_t* slots = smem + (size_t)warp * SPW * kSlot;
  uint8_t* xh = smem + (size_t)NW * SPW * kSlot;  // x rows (gate_up), then h rows (down)
  uint64_t* fb = full + warp * SPW;
  volatile int* abort_flag = &m.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NW * SPW; i++) mbar_init(&full[i], 1);
    m.abort = 0;
    fence_barrier_init();
  }
  pdl_enter();

  // ---- routing: every CTA routes the tokens itself (the same result everywhere); CTA 0
  // also writes the caller's topk outputs
  if (a.pre_routed) {
    for (int n = threadIdx.x; n < T * k; n += blockDim.x) {
      m.idx[n] = a.idx[n];
      m.w[n] = a.w[n];
    }
    if (threadIdx.x < T) m.sgate[threadIdx.x] = a.sgate ? a.sgate[threadIdx.x] : 1.f;
  } else {
    for (int t = warp; t < T; t += NW) {
      RouteArgs r = a.ra;
      r.idx = m.idx;
      r.w = m.w;
      r.sgate = a.has_sgate ? m.sgate : nullptr;
      if (blockIdx.x != 0) {
        r.idx_user = nullptr;
        r.w_user = nullptr;
      }
      routing::route_token<EPL>(r, t, lane);
      if (!a.has_sgate && lane == 0) m.sgate[t] = 1.f;
    }
  }
  {  // x rows, the gate_up operand
    const uint4* src = reinterpret_cast<const uint4*>(a.x);
    uint4* dst = reinterpret_cast<uint4*>(xh);
    for (int v = threadIdx.x; v < T * d / 8; v += blockDim.x) dst[v] = __ldg(src + v);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // distinct experts in order of first use, each with its token slots
    int U = 0;
    for (int t = 0; t < T; t++)
      for (int j = 0; j < k; j++) {
        const int e = m.idx[t * k + j];
        if (e < 0 || e >= a.E) {
          set_status(a.status, MOE_ERR_SHAPE);
          continue;
        }
        int u = 0;
        while (u < U && m.e[u] != e) u++;
        if (u == U) {
          m.e[U] = e;
          m.cnt[U] = 0;
          U++;
        }
        const int c = m.cnt[u];
        if (c >= kGemvMaxTokens) {  // a token chose the expert twice: not a top-k result
          set_status(a.status, MOE_ERR_SHAPE);
          continue;
        }
        m.tok[u][c] = t;
        m.row[u][c] = t * k + j;
        m.wt[u][c] = m.w[t * k + j];
        m.cnt[u] = c + 1;
      }
    if (a.Fs > 0) {
      m.e[U] = -1;
      m.cnt[U] = T;
      for (int t = 0; t < T; t++) {
        m.tok[U][t] = t;
        m.row[U][t] = R + t;
        m.wt[U][t] = 1.f;
      }
      U++;
    }
    m.n_ent = U;
  }
  __syncthreads();

  const int U = m.n_ent;
  const bool plain = a.ffn == MOE_FFN_PLAIN;
  const bool unfused = a.gu_layout == MOE_GU_UNFUSED;
  const int FJ = plain ? 16 : 8;  // features per gate_up job
  int JA = 0;                      // gate_up jobs of the whole grid
  for (int u = 0; u < U; u++) JA += (m.e[u] < 0 ? a.Fs : a.F) / FJ;
  const int G = gridDim.x;
  const int KSA = (d + kKS - 1) / kKS;                          // stages per job
  const int KSB = ((a.Fs > a.F ? a.Fs : a.F) + kKS - 1) / kKS;  // stages per unit
  const int NRB = (d + kRB - 1) / kRB;                          // row blocks
  const int ZB = NRB * U;                                       // down units
  const int64_t stride = (int64_t)G * NW;
  const int64_t ja0 = blockIdx.x + (int64_t)G * warp;  // this warp's first gate_up job
  const int nA = ja0 < JA ? (int)((JA - 1 - ja0) / stride + 1) : 0;
  const int64_t zb0 = ((((int64_t)blockIdx.x - JA) % G + G) % G) + (int64_t)G * warp;  // first down unit
  const int nB = zb0 < ZB ? (int)((ZB - 1 - zb0) / stride + 1) : 0;
  const int nsA = nA * KSA, n = nsA + nB * KSB;  // this warp's stages

  // ---- lane 0: the TMA loads of stage j into slot j % SPW
  JobCursor ci;
  int issued = 0;
  auto issue = [&](int j) {
    uint8_t* dst = slots + (size_t)(j % SPW) * kSlot;
    uint64_t* bar = &fb[j % SPW];
    mbar_arrive_expect_tx(bar, kSlot);
    if (j < nsA) {
      const int job = (int)(ja0 + stride * (j / KSA)), kb = (j % KSA) * kKB;
      ci.seek(m, a, FJ, job);
      const int e = m.e[ci.u], f0 = (job - ci.u0) * FJ;
      if (e < 0) {
        if (plain) tma_load_3d(&tm_sgu, bar, dst, 0, f0, kb);
        else tma_load_4d(&tm_sgu, bar, dst, 0, f0, kb, 0);
      } else if (unfused) {
        tma_load_4d(&tm_gu, bar, dst, 0, f0, kb, e);
        tma_load_4d(&tm_gu2, bar, dst + kSlot / 2, 0, f0, kb, e);
      } else if (plain) {
        tma_load_4d(&tm_gu, bar, dst, 0, f0, kb, e);
      } else {
        tma_load_5d(&tm_gu, bar, dst, 0, f0, kb, 0, e);
      }
    } else {
      const int jb = j - nsA;
      const int z = (int)(zb0 + stride * (jb / KSB)), kb = (jb % KSB) * kKB;
      const int e = m.e[z % U], n0 = (z / U) * kRB;
      if (e < 0) tma_load_3d(&tm_sdn, bar, dst, 0, n0, kb);
      else tma_load_4d(&tm_dn, bar, dst, 0, n0, kb, e);
    }
    issued = j + 1;
  };
  if (lane == 0)
    for (int j = 0; j < SPW && j < n; j++) issue(j);

  // Line of 128 bytes holding row r (< 16) of k-block kb in a slot: gated tiles are
  // [gate / up][kKB][8][64], the others [kKB][16][64]; the 128-byte swizzle XORs the
  // 16-byte chunk with the line index mod 8, which is r mod 8 in both.
  auto line_of = [&](bool gated, int kb, int r) { return gated ? ((r >> 3) * kKB + kb) * 8 + (r & 7) : kb * 16 + r; };
  // One stage: 16 k16 steps of mma.sync into four accumulator sets (step ks into set
  // ks mod 4, so that consecutive MMAs do not wait on each other).  A comes from the
  // swizzled tile by ldmatrix (lane l addresses row l mod 8 (+8 for matrices 1 and 3)
  // of k-chunk c0 (+1 for matrices 2 and 3)); B column g is the bf16 row `col` (null:
  // a zero column), read from element k0 on; K stops at kend.  Four steps' operands
  // are loaded before their four MMAs.
  const int lr = (lane & 7) + ((lane >> 3) & 1) * 8, lc = lane >> 4;  // this lane's ldmatrix row, chunk
  auto stage_mma = [&](float (&acc)[kAcc][4], const uint8_t* tile, bool gated, const uint8_t* col, int k0,
                       int kend) {
    const int steps = kend - k0 >= kKS ? kKS / 16 : (kend - k0) / 16;
    for (int s0 = 0; s0 < steps; s0 += 4) {
      uint32_t af[4][4], bf[4][2];
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const int ks = s0 + q;
        if (ks < steps) {
          const int kb = ks >> 2, c = (ks & 3) * 2 + lc;
          const uint8_t* p = tile + line_of(gated, kb, lr) * 128 + ((c ^ (lr & 7)) << 4);
          asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                       : "=r"(af[q][0]), "=r"(af[q][1]), "=r"(af[q][2]), "=r"(af[q][3])
                       : "r"(smem_u32(p)));
          bf[q][0] = bf[q][1] = 0;
          if (col) {
            const int kk = k0 + ks * 16;
            bf[q][0] = lds32(col + 2 * (kk + 2 * t4));
            bf[q][1] = lds32(col + 2 * (kk + 8 + 2 * t4));
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 4; q++)
        if (s0 + q < steps) mma_16816(acc[q], af[q][0], af[q][1], af[q][2], af[q][3], bf[q][0], bf[q][1]);
    }
  };

  // ---- gate_up jobs: lane (g, t4) ends with rows g and g + 8 (gate and up of feature
  // f0 + g, or plain features f0 + g and f0 + g + 8) for slots 2 t4 and 2 t4 + 1
  JobCursor cc;
  float acc[kAcc][4], v[4];
  auto clear = [&] {
#pragma unroll
    for (int q = 0; q < kAcc; q++) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.f;
  };
  auto total = [&] {  // the four sets, added in a fixed order
#pragma unroll
    for (int i = 0; i < 4; i++) v[i] = (acc[0][i] + acc[1][i]) + (acc[2][i] + acc[3][i]);
  };
  bool ok = true;
  for (int j = 0; j < nsA; j++) {
    const bool have = __all_sync(0xffffffffu, wait_tile(&fb[j % SPW], (j / SPW) & 1, abort_flag, a.status));
    ok = ok && have;
    const int job = (int)(ja0 + stride * (j / KSA)), sl = j % KSA;
    cc.seek(m, a, FJ, job);
    const int u = cc.u, e = m.e[u], cnt = m.cnt[u], f0 = (job - cc.u0) * FJ;
    if (sl == 0) clear();
    if (have) {
      const uint8_t* col = g < cnt ? xh + (size_t)m.tok[u][g] * 2 * d : nullptr;
      stage_mma(acc, slots + (size_t)(j % SPW) * kSlot, !plain, col, sl * kKS, d);
    }
    __syncwarp();
    if (lane == 0 && j + SPW < n && !*abort_flag) issue(j + SPW);
    if (sl != KSA - 1) continue;
    total();
    if (ok) {
#pragma unroll
      for (int h2 = 0; h2 < 2; h2++) {
        const int s = 2 * t4 + h2;  // slot
        if (s >= cnt) continue;
        const float wi = (e >= 0 && a.weigh_inputs) ? m.wt[u][s] : 1.f;
        uint16_t* hrow = a.h + (int64_t)m.row[u][s] * a.Fmax;
        if (!plain) {
          const int f = f0 + g;
          float bg = 0.f, bu = 0.f;
          if (e >= 0) {
            const GuBias gb = gu_bias(a.gu_layout, a.F, e, a.gate_up_bias, a.gate_bias);
            if (gb.g) bg = bf16_to_f32(gb.g[(int64_t)gb.stride * f]);
            if (gb.u) bu = bf16_to_f32(gb.u[(int64_t)gb.stride * f]);
          }
          hrow[f] = f32_to_bf16_rn(gated_act_bf16(a.act, fmaf(wi, v[h2], bg), fmaf(wi, v[2 + h2], bu)));
        } else {
#pragma unroll
          for (int hi = 0; hi < 2; hi++) {
            const int f = f0 + g + 8 * hi;
            const float b = (e >= 0 && a.gate_up_bias) ? bf16_to_f32(a.gate_up_bias[(int64_t)e * a.F + f]) : 0.f;
            hrow[f] = f32_to_bf16_rn(plain_act_bf16(a.act, fmaf(wi, v[2 * hi + h2], b)));
          }
        }
      }
    }
    ok = true;
  }

  // ---- publish this CTA's h features, wait for every CTA's, stage all h rows
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(a.done, 1);
    if (ld_acquire_gpu(a.done) < G) {
      const uint64_t t0 = global_timer();
      while (ld_acquire_gpu(a.done) < G) {
        if (*abort_flag) break;
        if (global_timer() - t0 > kTimeoutNs) {
          *abort_flag = 1;
          set_status(a.status, MOE_ERR_TIMEOUT);
          break;
        }
        __nanosleep(32);
      }
    }
  }
  __syncthreads();
  {  // routed rows [R][F], then the shared expert's [T][Fs]
    const int vf = a.F / 8, vs = a.Fs / 8;
    uint4* hs = reinterpret_cast<uint4*>(xh);
    for (int v = threadIdx.x; v < R * vf; v += blockDim.x)
      hs[v] = __ldcg(reinterpret_cast<const uint4*>(a.h + (int64_t)(v / vf) * a.Fmax) + v % vf);
    for (int v = threadIdx.x; v < T * vs; v += blockDim.x)
      hs[R * vf + v] = __ldcg(reinterpret_cast<const uint4*>(a.h + (int64_t)(R + v / vs) * a.Fmax) + v % vs);
  }
  __syncthreads();

  // ---- down units: lane (g, t4) ends with output rows n0 + g and n0 + g + 8 for slots
  // 2 t4 and 2 t4 + 1
  ok = true;
  for (int j = nsA; j < n; j++) {
    const bool have = __all_sync(0xffffffffu, wait_tile(&fb[j % SPW], (j / SPW) & 1, abort_flag, a.status));
    ok = ok && have;
    const int jb = j - nsA, sl = jb % KSB;
    const int z = (int)(zb0 + stride * (jb / KSB)), u = z % U, rb = z / U;
    const int e = m.e[u], cnt = m.cnt[u], ku = e < 0 ? a.Fs : a.F, n0 = rb * kRB;
    if (sl == 0) clear();
    if (have) {
      const uint8_t* col = nullptr;
      if (g < cnt) {
        const int row = m.row[u][g];
        col = xh + (e < 0 ? (size_t)(R * a.F + (row - R) * a.Fs) * 2 : (size_t)row * a.F * 2);
      }
      stage_mma(acc, slots + (size_t)(j % SPW) * kSlot, false, col, sl * kKS, ku);
    }
    __syncwarp();
    if (lane == 0 && j + SPW < n && !*abort_flag) issue(j + SPW);
    if (sl != KSB - 1) continue;
    total();
    if (ok) {
#pragma unroll
      for (int hi = 0; hi < 2; hi++)
#pragma unroll
        for (int h2 = 0; h2 < 2; h2++) {
          const int s = 2 * t4 + h2, nn = n0 + g + 8 * hi;
          if (s >= cnt || nn >= d) continue;
          const float b = (e >= 0 && a.down_bias) ? bf16_to_f32(a.down_bias[(int64_t)e * d + nn]) : 0.f;
          const float wt = (e < 0 || a.weigh_inputs) ? 1.f : m.wt[u][s];
          a.Y[(int64_t)m.row[u][s] * d + nn] = f32_to_bf16_rn((v[2 * hi + h2] + b) * wt);
        }
    }
    ok = true;
    // the last unit of this row block combines it, slot order per token
    __threadfence();
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atomicAdd(a.rb_done + rb, 1) == U - 1;
    if (__shfl_sync(0xffffffffu, last, 0) && !*abort_flag) {
      __threadfence();
      for (int o = lane; o < T * kRB; o += 32) {
        const int t = o / kRB, nn = n0 + o % kRB;
        if (nn >= d) continue;
        float y = 0.f;
        for (int jj = 0; jj < k; jj++) y += bf16_to_f32(__ldcg(a.Y + (int64_t)(t * k + jj) * d + nn));
        if (a.Fs > 0) y += m.sgate[t] * bf16_to_f32(__ldcg(a.Y + (int64_t)(R + t) * d + nn));
        if (a.shared_output) y += bf16_to_f32(a.shared_output[(int64_t)t * d + nn]);
        a.y[(int64_t)t * d + nn] = f32_to_bf16_rn(y);
      }
    }
  }

  // every load this warp issued has landed before the CTA may exit
  if (lane == 0) {
    for (int j = issued > SPW ? issued - SPW : 0; j < issued; j++) {
      const uint64_t t0 = global_timer();
      while (!mbar_try_wait(&fb[j % SPW], (j / SPW) & 1) && global_timer() - t0 < kTimeoutNs) {
      }
    }
  }
}

// ---------------------------------------------------------------- host side

// bf16 tensor map, 128-byte swizzle; dims[0] = 64 (one 128-byte line), strides in bytes.
bool gmap(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
          const uint32_t* box) {
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

// A weight matrix of `rows` rows of K elements (row pitch `pitch` bytes) as {64, rows,
// K / 64 [, outer]}: a box of `box_rows` rows by kKB k-blocks lands as [kKB][box_rows][64].
bool map_tiles(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t pitch, uint32_t box_rows,
               uint64_t outer, uint64_t outer_stride) {
  const uint64_t dims[4] = {64, rows, K / 64, outer};
  const uint64_t strides[3] = {pitch, 128, outer_stride};
  const uint32_t box[4] = {64, box_rows, kKB, 1};
  return gmap(m, base, outer > 0 ? 4 : 3, dims, strides, box);
}

// A fused gate / up stack: {64, F, d / 64, 2 [, E]}, the gate (0) / up (1) index with
// its own stride; a box of 8 features lands as [gate, up][kKB][8][64].
bool map_fused(CUtensorMap* m, const void* base, uint64_t d, uint64_t F, bool interleaved, uint64_t E) {
  const uint64_t row = interleaved ? 2 * d * 2 : d * 2, gu = interleaved ? d * 2 : F * d * 2;
  const uint64_t dims[5] = {64, F, d / 64, 2, E};
  const uint64_t strides[4] = {row, 128, gu, 2 * F * d * 2};
  const uint32_t box[5] = {64, 8, kKB, 2, 1};
  return gmap(m, base, E > 0 ? 5 : 4, dims, strides, box);
}

template <int EPL>
cudaError_t launch_epl(const CUtensorMap (&tm)[5], const GemvArgs& a, int num_sms, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(gemv_ffn_kernel<EPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, a.smem_bytes);
  if (e != cudaSuccess) return e;
  return launch_coop_pdl(gemv_ffn_kernel<EPL>, dim3(num_sms), dim3(a.warps * 32), (size_t)a.smem_bytes, st, tm[0],
                         tm[1], tm[2], tm[3], tm[4], a);
}

}  // namespace

cudaError_t launch_gemv_ffn(const GemvArgs& a, int num_sms, cudaStream_t st) {
  if (a.T < 1 || a.T > kGemvMaxTokens || a.warps < 4 || a.warps > kGemvMaxWarps) return cudaErrorInvalidValue;
  if (a.d % 64 || a.F % 64 || a.Fs % 64) return cudaErrorInvalidValue;
  const uint64_t d = a.d, F = a.F, Fs = a.Fs, E = a.E;
  const bool plain = a.ffn == MOE_FFN_PLAIN;
  // 0: routed gate_up (unfused: the gate rows), 1: unfused up rows, 2: shared gate_up,
  // 3: routed down, 4: shared down; maps a call does not read are copies of map 0
  CUtensorMap tm[5];
  bool ok;
  if (plain) {
    ok = map_tiles(&tm[0], a.gate_up, d, F, d * 2, 16, E, F * d * 2);
  } else if (a.gu_layout == MOE_GU_UNFUSED) {
    ok = map_tiles(&tm[0], a.gate, d, F, d * 2, 8, E, F * d * 2) &&
         map_tiles(&tm[1], a.gate_up, d, F, d * 2, 8, E, F * d * 2);
  } else {
    ok = map_fused(&tm[0], a.gate_up, d, F, a.gu_layout == MOE_GU_INTERLEAVED, E);
  }
  if (ok && Fs > 0) {
    ok = plain ? map_tiles(&tm[2], a.sh_gate_up, d, Fs, d * 2, 16, 0, 0)
               : map_fused(&tm[2], a.sh_gate_up, d, Fs, a.gu_layout == MOE_GU_INTERLEAVED, 0);
    ok = ok && map_tiles(&tm[4], a.sh_down, Fs, d, Fs * 2, kRB, 0, 0);
  }
  ok = ok && map_tiles(&tm[3], a.down, F, d, F * 2, kRB, E, d * F * 2);
  if (!ok) return cudaErrorInvalidValue;
  if (a.gu_layout != MOE_GU_UNFUSED || plain) tm[1] = tm[0];
  if (Fs == 0) tm[2] = tm[4] = tm[0];
  const int epl = a.pre_routed ? 1 : (a.E + 31) / 32;
  if (epl <= 1) return launch_epl<1>(tm, a, num_sms, st);
  if (epl <= 2) return launch_epl<2>(tm, a, num_sms, st);
  if (epl <= 4) return launch_epl<4>(tm, a, num_sms, st);
  if (epl <= 8) return launch_epl<8>(tm, a, num_sms, st);
  return cudaErrorInvalidValue;
}

}  // namespace moe
