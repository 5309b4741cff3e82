// lowm.cu — QLoRA linear forward for a few tokens (M <= 16) on a large weight:
//   Y = X W'^T + s (X A^T) B^T,  W' = NF4-dequantised frozen weight
// ("QLoRA" encyclopedia entry, tonho.wtf, section "como funciona": the
// frozen weight is stored in NF4 and turned back into BFloat16 only where it
// is used; the adapters stay 16-bit).
//
// At M <= 16 the product does at most 64 flops per byte of NF4 codes, so the
// weight stream and the nibble-to-bf16 lookups bound it, not the tensor
// pipe.  This kernel therefore keeps the dequantised weight in registers:
// every lane turns its own codes into bf16 pairs with byte-permute lookups
// and hands them straight to register-operand MMAs (m16n8k16, fp32
// accumulate).  The weight never goes back to shared memory.
//
// Work unit: 128 rows of W (one 16-row slice per warp) x 256 input features
// (four 64-element blocks; lane t of each quad owns block t, so each lane
// builds one lookup table per row and block).  The contraction slots of each
// MMA step j take, per lane, the 8 features of chunk (j ^ c_t) of that lane's
// own block, c_t = 5t mod 8; the token fragments read X at the same features,
// so the permutation cancels.  The lane-dependent chunk order makes every
// shared-memory read conflict-free: the 8 lanes of each quarter warp (two
// rows g, four blocks t) hit 8 different 16-byte bank groups.
//
// U = X A^T (fp32) comes from the rank-r kernel launched just before this one
// (programmatic dependent launch: the main loop below runs beside it).
//
// Lane 0 of warp 0 streams each unit's codes (one 128 x 128-byte TMA box) and
// its X slice (four 64-feature boxes; rows past M and features past K arrive
// as zeros) into a shared-memory ring of four stages, two
// units ahead of the unit being computed.  No warp is set aside for the
// copies, so every warp has the full register budget.
//
// The units (row tile major, K chunk minor) are cut into equal contiguous
// ranges, one per persistent CTA.  A range spans at most two row tiles (the
// CTA count is at least the tile count); the CTA writes one fp32 partial per
// tile it touches and counts it in on the tile's counter.  The CTA that counts
// a tile's last partial finishes the tile: it adds the partials in CTA order
// (a fixed order: results are deterministic), adds s U B^T in fp32 and rounds
// once.
#include "kernels.h"

namespace qnf4 {

namespace {

constexpr int kLowmWarps = kLowmThreads / 32;
constexpr int kLowmAhead = 2;                     // units in flight ahead of the one computed
constexpr uint32_t kLowmCodes = kLowmRows * 128;  // 16 KB: 128 rows x 256 codes, or 32 A rows x 256 bf16

template <int NT>
struct LowmPlan {
  static constexpr uint32_t kXBox = 8 * NT * 128;  // {64 features, 8 NT tokens} bf16
  static constexpr uint32_t kStage = kLowmCodes + 4 * kXBox;
  static constexpr int kStages = 4;  // two CTAs per SM
  static constexpr uint32_t kBarOff = kStages * kStage;
  static constexpr uint32_t kSmem = kBarOff + 2 * kStages * 8 + 16 + 1024;
  static_assert(kStages > kLowmAhead, "ring must hold the units in flight plus the one computed");
};

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

__device__ __forceinline__ int64_t unit_start(int64_t c, int64_t units, int ctas) { return c * units / ctas; }

// CTA whose range holds unit u: the largest c with floor(c * L / P) <= u.
__device__ __forceinline__ int cta_of_unit(int64_t u, int64_t units, int ctas) {
  return static_cast<int>(((u + 1) * ctas - 1) / units);
}

__device__ __forceinline__ int64_t lowm_units(const LowmArgs& a) {
  return static_cast<int64_t>(a.tiles + a.atiles) * a.kc;
}

// Whether this warp has rows in `tile`: all 16 rows of its slice exist (N is
// a multiple of 64).
__device__ __forceinline__ bool warp_rows_valid(const LowmArgs& a, int tile, int warp) {
  return tile * kLowmRows + warp * 16 + 16 <= a.N;
}

// Block constants of rows g and g + 8 of this warp's slice, block t of the
// unit's chunk (zero where the block does not exist: the table is then 0).
struct UnitConsts {
  uint32_t ca, cb;
  float sa, sb;
};

__device__ __forceinline__ void load_consts(const LowmArgs& a, int tile, int kci, int warp, int g, int t,
                                            UnitConsts& c) {
  const int blk = kci * 4 + t;
  const int kb = a.K >> 6;
  c.ca = c.cb = 0;
  c.sa = c.sb = 0.0f;
  if (tile >= a.tiles || blk >= kb || !warp_rows_valid(a, tile, warp)) return;
  const int64_t ia = (static_cast<int64_t>(tile) * kLowmRows + warp * 16 + g) * kb + blk, ib = ia + 8 * kb;
  c.ca = __ldg(a.c8 + ia);
  c.cb = __ldg(a.c8 + ib);
  c.sa = __ldg(a.s2 + (ia >> 8));
  c.sb = __ldg(a.s2 + (ib >> 8));
}

// Lane 0 of warp 0: issue the copies of unit `i` of this CTA's range into
// stage i % kStages once the eight warps have released its previous use.
template <int NT>
__device__ __forceinline__ bool lowm_issue(const CUtensorMap* tm_codes, const CUtensorMap* tm_x, uint8_t* smem,
                                           uint64_t* full, uint64_t* empty, int i, int tile, int kci,
                                           const WaitCtx& wc) {
  using P = LowmPlan<NT>;
  const int s = i % P::kStages;
  if (i >= P::kStages && !mbar_wait(&empty[s], ((i / P::kStages) & 1) ^ 1, wc)) return false;
  uint8_t* st = smem + s * P::kStage;
  mbar_arrive_expect_tx(&full[s], kLowmCodes + 4 * P::kXBox);
  tma_load_2d(st, tm_codes, &full[s], kci * 128, tile * kLowmRows);
#pragma unroll
  for (int b = 0; b < 4; ++b) tma_load_2d(st + kLowmCodes + b * P::kXBox, tm_x, &full[s], kci * 256 + b * 64, 0);
  return true;
}

// The CTAs whose ranges hold units of row tile `tile`: c0 .. c1.
__device__ __forceinline__ void tile_ctas(const LowmArgs& a, int tile, int& c0, int& c1) {
  const int64_t units = lowm_units(a);
  c0 = cta_of_unit(static_cast<int64_t>(tile) * a.kc, units, a.ctas);
  c1 = cta_of_unit(static_cast<int64_t>(tile + 1) * a.kc - 1, units, a.ctas);
}

// Row stride of the staged B tile in shared memory: 128 bytes of a row (r <=
// 64 bf16) plus 16 of padding, so the 16-byte reads of the eight lanes of a
// quarter warp (eight consecutive rows) fall in different bank groups.
constexpr int kSbStride = 144;

// Y rows of `tile` = the sum of its partials in CTA order + s U B^T (fp32,
// one rounding), by the CTA that wrote the tile's last partial.  Thread:
// row = tid % 128, tokens (tid / 128) * mpad/2 ..; su holds U's columns of the
// tile's group member for the M tokens, sb the tile's rows of B.
template <int NT>
__device__ void finish_tile(const LowmArgs& a, int tile, const float* su, const uint8_t* sb) {
  constexpr int kMpad = 8 * NT;
  constexpr int kHalf = kMpad / 2;
  const int row = threadIdx.x & (kLowmRows - 1);
  const int m0 = (threadIdx.x >> 7) * kHalf;
  const int n = tile * kLowmRows + row;
  if (n >= a.N || m0 >= a.M) return;
  int c0, c1;
  tile_ctas(a, tile, c0, c1);
  const int64_t units = lowm_units(a);
  float y[kHalf];
#pragma unroll
  for (int e = 0; e < kHalf; ++e) y[e] = 0.0f;
#pragma unroll 2
  for (int c = c0; c <= c1; ++c) {
    const int first = static_cast<int>(unit_start(c, units, a.ctas) / a.kc);
    const float* src = a.part + ((static_cast<int64_t>(c) * 2 + (tile == first ? 0 : 1)) * kLowmRows + row) * kMpad + m0;
#pragma unroll
    for (int e = 0; e < kHalf; e += 4) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(src + e));
      y[e] = __fadd_rn(y[e], v.x);
      y[e + 1] = __fadd_rn(y[e + 1], v.y);
      y[e + 2] = __fadd_rn(y[e + 2], v.z);
      y[e + 3] = __fadd_rn(y[e + 3], v.w);
    }
  }
  float lo[kHalf];
#pragma unroll
  for (int e = 0; e < kHalf; ++e) lo[e] = 0.0f;
  const uint8_t* brow = sb + row * kSbStride;
  for (int j8 = 0; j8 < a.r / 8; ++j8) {
    const uint4 bv = *reinterpret_cast<const uint4*>(brow + j8 * 16);
    const uint32_t w[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float b = __uint_as_float(e & 1 ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
#pragma unroll
      for (int mm = 0; mm < kHalf; ++mm) lo[mm] = fmaf(su[(m0 + mm) * 64 + 8 * j8 + e], b, lo[mm]);
    }
  }
#pragma unroll
  for (int mm = 0; mm < kHalf; ++mm) {
    const int m = m0 + mm;
    if (m < a.M) {
      const float v = y[mm] + a.s * lo[mm];
      const int64_t o = static_cast<int64_t>(m) * a.N + n;
      if (a.y_f32) reinterpret_cast<float*>(a.Y)[o] = v;
      else reinterpret_cast<uint16_t*>(a.Y)[o] = bf16_bits(v);
    }
  }
}

template <int NT>
__global__ void __launch_bounds__(kLowmThreads, 2)
    lowm_fwd_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                    const LowmArgs a) {
  using P = LowmPlan<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::kBarOff);
  uint64_t* empty = full + P::kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + P::kStages);
  int* last_flag = const_cast<int*>(abort_flag) + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool issuer = threadIdx.x == 0;

  const int64_t units = lowm_units(a);
  const int64_t u_beg = unit_start(blockIdx.x, units, a.ctas);
  const int count = static_cast<int>(unit_start(blockIdx.x + 1, units, a.ctas) - u_beg);
  const int tile0 = static_cast<int>(u_beg / a.kc);
  const int kci0 = static_cast<int>(u_beg - static_cast<int64_t>(tile0) * a.kc);

  if (issuer) {
    for (int s = 0; s < P::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kLowmWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_x);
  }
  __syncthreads();
  const WaitCtx wc{abort_flag, a.status};
  // Programmatic dependent launch: the kernel launched just before this one
  // computes U (and clears the tile counters); the codes, constants and X
  // come from earlier kernels, complete when it let this one start.  So the
  // main loop runs beside it, and the wait comes before U and the counters
  // are touched (and before this kernel lets its own dependents start).
  const Nf4Mean wmean = nf4_load_mean(a.mean);

  // Copy issue state (lane 0 of warp 0 only).
  int issued = 0, itile = tile0, ikci = kci0;
  bool ok = true;
  auto issue_next = [&]() {
    ok = lowm_issue<NT>(&tm_codes, &tm_x, smem, full, empty, issued, itile, ikci, wc);
    if (ok) {
      ++issued;
      if (++ikci == a.kc) {
        ikci = 0;
        ++itile;
      }
    }
  };
  if (issuer) {
    while (ok && issued < count && issued < kLowmAhead) issue_next();
  }

  const int g = lane >> 2, t = lane & 3;
  const uint32_t ct = (5u * static_cast<uint32_t>(t)) & 7u;
  // Byte offsets, within a 128-byte swizzled row of phase g, of codes word
  // (j ^ ct) of block t (XOR j << 2 for step j), and of X chunk (j ^ ct)
  // (XOR j << 4 for step j).
  const uint32_t code_off = ((static_cast<uint32_t>(2 * t) ^ static_cast<uint32_t>(g)) << 4) ^ (ct << 2);
  const uint32_t chunk_off = (ct ^ static_cast<uint32_t>(g)) << 4;

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;

  int tile = tile0, kci = kci0;
  UnitConsts cur;
  load_consts(a, tile, kci, warp, g, t, cur);
  for (int i = 0; i < count; ++i) {
    int ntile = tile, nkci = kci + 1;
    if (nkci == a.kc) {
      nkci = 0;
      ++ntile;
    }
    const bool more = i + 1 < count;
    if (issuer && ok && issued < count) issue_next();
    const int s = i % P::kStages;
    if (!mbar_wait_all(&full[s], (i / P::kStages) & 1, wc)) break;
    const uint8_t* st = smem + s * P::kStage;
    // X box of this lane's block; token row 8n + g has phase g.
    const uint8_t* xs = st + kLowmCodes + t * P::kXBox + g * 128;
    if (warp_rows_valid(a, tile, warp)) {
      const Nf4Lut la = nf4_make_lut(a.tab, nf4_block_scale(cur.ca, cur.sa, wmean));
      const Nf4Lut lb = nf4_make_lut(a.tab, nf4_block_scale(cur.cb, cur.sb, wmean));
      // The next unit's constants load into `cur` (dead from here on) and
      // have a whole unit of work to arrive.
      if (more) load_consts(a, ntile, nkci, warp, g, t, cur);
      // rows warp*16 + g and + 8, both of phase g
      const uint8_t* ra = st + (warp * 16 + g) * 128;
      uint32_t wa[8], wb[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t o = code_off ^ (static_cast<uint32_t>(j) << 2);
        wa[j] = lds32(ra + o);
        wb[j] = lds32(ra + 1024 + o);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 oa = nf4_lookup8(wa[j], la);
        const uint4 ob = nf4_lookup8(wb[j], lb);
        const uint32_t xo = chunk_off ^ (static_cast<uint32_t>(j) << 4);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint4 xv = lds128(xs + n * 1024 + xo);
          mma_16816(acc[n], oa.x, ob.x, oa.y, ob.y, xv.x, xv.y);
          mma_16816(acc[n], oa.z, ob.z, oa.w, ob.w, xv.z, xv.w);
        }
      }
    } else if (more) {
      load_consts(a, ntile, nkci, warp, g, t, cur);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    // Last unit of this tile in the range: write the partial, restart.
    if (!more || ntile != tile) {
      const int slot = tile == tile0 ? 0 : 1;
      constexpr int kMpad = 8 * NT;  // == a.mpad
      float* dst = a.part + ((static_cast<int64_t>(blockIdx.x) * 2 + slot) * kLowmRows + warp * 16 + g) * kMpad +
                   2 * t;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        *reinterpret_cast<float2*>(dst + 8 * n) = make_float2(acc[n][0], acc[n][1]);
        *reinterpret_cast<float2*>(dst + 8 * kMpad + 8 * n) = make_float2(acc[n][2], acc[n][3]);
        acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
      }
    }
    tile = ntile;
    kci = nkci;
  }
  // After a timeout, let copies still in flight land before the CTA exits
  // (after a normal run every stage's last phase has completed already).
  if (issuer) {
    for (int i = max(0, issued - P::kStages); i < issued; ++i)
      mbar_drain(&full[i % P::kStages], (i / P::kStages) & 1, a.status);
  }

  grid_dependency_wait();  // U and the cleared tile counters are complete and visible
  grid_dependents_launch();
  if (count <= 0) return;

  // Each row tile this CTA wrote a partial of (at most two): count the
  // partial in; the CTA that counts the tile's last one finishes the tile.
  __threadfence();  // this thread's partial stores, before the count
  __syncthreads();
  // The ring is idle now: U of the member, [mpad][64] fp32, then the tile's
  // rows of B, [128][kSbStride bytes].
  float* su = reinterpret_cast<float*>(smem);
  uint8_t* sb = smem + 8 * NT * 64 * 4;
  const int tile_last = static_cast<int>((u_beg + count - 1) / a.kc);
  for (int tl = tile0; tl <= tile_last; ++tl) {
    if (threadIdx.x == 0) {
      int c0, c1;
      tile_ctas(a, tl, c0, c1);
      const unsigned prev = atomicAdd(a.tile_count + tl, 1u);
      *last_flag = prev == static_cast<unsigned>(c1 - c0) ? 1 : 0;
      __threadfence();  // the other CTAs' partials, before this CTA reads them
    }
    __syncthreads();
    if (*last_flag) {
      // U of the member and the tile's rows of B into shared memory, 16-byte
      // loads (rows of U and the member's column offset are multiples of 16
      // floats; rows of B are r <= 64 bf16), all of a thread's in flight
      // before any is stored.
      const int mem = group_member(a.grp_end, a.groups, tl * kLowmRows);
      constexpr int kUq = 8 * NT * 16, kBq = kLowmRows * 8;
      constexpr int kUn = (kUq + kLowmThreads - 1) / kLowmThreads, kBn = kBq / kLowmThreads;
      float4 uv[kUn];
      uint4 bq[kBn];
#pragma unroll
      for (int q = 0; q < kUn; ++q) {
        const int e4 = static_cast<int>(threadIdx.x) + q * kLowmThreads;
        const int m = e4 >> 4, jj = (e4 & 15) * 4;
        uv[q] = (e4 < kUq && m < a.M && jj < a.r)
                    ? __ldcg(reinterpret_cast<const float4*>(a.U + static_cast<int64_t>(m) * a.ra + mem * a.r + jj))
                    : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
#pragma unroll
      for (int q = 0; q < kBn; ++q) {
        const int e8 = static_cast<int>(threadIdx.x) + q * kLowmThreads;
        const int rw = e8 >> 3, j8 = e8 & 7;
        const int64_t n = static_cast<int64_t>(tl) * kLowmRows + rw;
        bq[q] = (n < a.N && j8 < a.r / 8) ? __ldg(reinterpret_cast<const uint4*>(a.B + n * a.r) + j8)
                                          : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int q = 0; q < kUn; ++q) {
        const int e4 = static_cast<int>(threadIdx.x) + q * kLowmThreads;
        if (e4 < kUq) reinterpret_cast<float4*>(su)[e4] = uv[q];
      }
#pragma unroll
      for (int q = 0; q < kBn; ++q) {
        const int e8 = static_cast<int>(threadIdx.x) + q * kLowmThreads;
        *reinterpret_cast<uint4*>(sb + (e8 >> 3) * kSbStride + (e8 & 7) * 16) = bq[q];
      }
      __syncthreads();
      finish_tile<NT>(a, tl, su, sb);
    }
    __syncthreads();
  }
}

template <int NT>
static cudaError_t launch_lowm_impl(const CUtensorMap& tm_codes, const CUtensorMap& tm_x, const LowmArgs& a,
                                    cudaStream_t stream) {
  static bool attr_set = false;  // benign race: setting the same value twice is harmless
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(lowm_fwd_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(LowmPlan<NT>::kSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_kernel(lowm_fwd_kernel<NT>, dim3(a.ctas), dim3(kLowmThreads), LowmPlan<NT>::kSmem, stream,
                       dim3(1, 1, 1), tm_codes, tm_x, a);
}

}  // namespace

cudaError_t launch_lowm_fwd(const CUtensorMap& tm_codes, const CUtensorMap& tm_x, const LowmArgs& a,
                            cudaStream_t stream) {
  switch (a.mpad) {
    case 8: return launch_lowm_impl<1>(tm_codes, tm_x, a, stream);
    case 16: return launch_lowm_impl<2>(tm_codes, tm_x, a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qnf4
