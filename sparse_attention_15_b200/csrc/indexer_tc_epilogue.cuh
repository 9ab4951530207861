// A fragment of index_scores_tc_kernel's body (indexer_tc.cu): the epilogue role.  The kernel
// includes it twice, once under the register split (inside the branch of a warpgroup,
// after its setmaxnreg) and once in the flat role dispatch of the kernels without the
// split, so that ptxas sees the same code in each form; lambdas or helper functions
// changed its register allocation.
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - kEpiWarp0;
    const int quad = warp & 3;
    const int group = ew >> 2;
    const int col0 = group * C::COLS_PER_WARP;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
    const float ninf = __int_as_float(0xff800000);
    UnitIter it(cta);
    uint32_t ci = 0;
    bool ok = true;
    // Filter mode: the candidates of each of this warp's queries found in one key tile are
    // written when that query comes round again in the next tile (or at the end of the
    // unit): the list position comes from a global atomicAdd issued when the scores are
    // ready, and its round trip overlaps the next tile's work instead of stalling this one.
    constexpr int QW = C::CL ? 1 : (C::COLS_PER_WARP / C::HI);  // queries per warp and tile
    struct Pending {
      uint32_t bal, key;
      int t, base;
      size_t off;
    };
    Pending pend[QW];
    uint32_t tau_q[QW];
#pragma unroll
    for (int q = 0; q < QW; ++q) pend[q].bal = 0u;
    const uint32_t lt_mask = (1u << lane) - 1u;
    auto flush = [&](Pending& p) {  // p.bal is warp-uniform
      if (p.bal) {
        const int base = __shfl_sync(0xffffffffu, p.base, 0);
        const int pos = base + __popc(p.bal & lt_mask);
        if (((p.bal >> lane) & 1u) && pos < a.cand_cap)
          a.cand[p.off + pos] = make_uint2(p.key, (uint32_t)p.t);
        p.bal = 0u;
      }
    };
    while (ok && it.next(a, C::NQ, ncta)) {
      const int s_base = it.qb * C::NQ;
      if constexpr (FILTER) {
#pragma unroll
        for (int q = 0; q < QW; ++q) {
          flush(pend[q]);
          const int sq = s_base + col0 / C::HI + q;
          tau_q[q] = sq < a.S ? __ldg(a.tau + (size_t)it.b * a.S + sq) : 0xffffffffu;
        }
      }
      // the head weights of this warp's columns are the same for every key tile of the unit
      // and every lane: read once per unit (broadcast float4 loads) and kept in registers
      // (the filter form, with more state per thread, reads them per tile instead)
      constexpr bool WREG = kSplit;
      float wq[WREG ? C::COLS_PER_WARP : 1];
      const float4* wunit = reinterpret_cast<const float4*>(
          C::CL ? a.w : a.w + ((size_t)it.b * a.S + s_base) * C::HI);
      if constexpr (WREG) {
        const float4* wcol = reinterpret_cast<const float4*>(
            a.w + ((size_t)it.b * a.S + s_base) * C::HI + col0);
#pragma unroll
        for (int i = 0; i < C::COLS_PER_WARP; i += 4) {
          // columns past the last query of a ragged block: no weight (never used)
          const float4 w4 = s_base + (col0 + i) / C::HI < a.S ? __ldg(wcol + i / 4)
                                                             : make_float4(0.f, 0.f, 0.f, 0.f);
          wq[i] = w4.x; wq[i + 1] = w4.y; wq[i + 2] = w4.z; wq[i + 3] = w4.w;
        }
      }
      for (int kt = it.k0; kt < it.k1; ++kt) {
        const int ab = ci % C::NACC;
        if (!warp_wait(&acc_full[ab], (ci / C::NACC) & 1)) { ok = false; break; }
        tc_fence_after();
        const int tcol = kt * kTileM + quad * 32 + lane;  // output column
        const int t = kt * a.kstride * kTileM + quad * 32 + lane;  // key position
        constexpr int NCH = C::COLS_PER_WARP / 16;
        // 16-column TMEM reads, double-buffered (chunk cc+1 in flight while chunk cc is
        // reduced) unless the weights held in registers leave no room for the second buffer.
        // A query's HI columns span HI/16 chunks; its four FMA chains carry over.
        constexpr int NBUF = (kSplit && C::COLS_PER_WARP > 32) ? 1 : 2;
        uint32_t rb[NBUF][16];
        tmem_ld16(t_lane + ab * C::ACC_COLS + col0, rb[0]);
        tmem_wait_ld();
        // four independent FMA chains (heads h % 4) as two packed float32 pairs
        unsigned long long acc01 = pack2(0.f, 0.f), acc23 = pack2(0.f, 0.f);
#pragma unroll
        for (int cc = 0; cc < NCH; ++cc) {
          if (cc + 1 < NCH) {
            if constexpr (NBUF == 2)
              tmem_ld16(t_lane + ab * C::ACC_COLS + col0 + (cc + 1) * 16, rb[(cc + 1) & 1]);
          } else {
            // every column of this accumulator has been read: hand it back to the MMA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
          }
          const uint32_t* r = rb[NBUF == 2 ? (cc & 1) : 0];
          const int c0 = col0 + cc * 16;     // first column of the chunk
          if constexpr (C::CL) {
            // eight queries per chunk: score = scale * (D[t, hi] + D[t, lo])
            const int sq = s_base + c0 / 2;
            float* op = a.scores + ((size_t)it.b * a.S + sq) * a.ldT + tcol;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              if (sq + q < a.S && t < a.T) {
                float v = (__uint_as_float(r[2 * q]) + __uint_as_float(r[2 * q + 1])) * a.scale;
                if (RELU == 1) v = fmaxf(v, 0.f);
                op[(size_t)q * a.ldT] = (t <= sq + q + a.q_off) ? v : ninf;
              }
            }
          } else {
            const int j = c0 / C::HI;          // query within the block
            const int s = s_base + j;
            if (s < a.S) {  // ragged tail of the last block (warp-uniform)
#pragma unroll
              for (int h = 0; h < 16; h += 4) {
                float4 w4;
                if constexpr (WREG)
                  w4 = make_float4(wq[cc * 16 + h], wq[cc * 16 + h + 1], wq[cc * 16 + h + 2],
                                   wq[cc * 16 + h + 3]);
                else
                  w4 = __ldg(wunit + (c0 + h) / 4);
                float d0 = __uint_as_float(r[h + 0]);
                float d1 = __uint_as_float(r[h + 1]);
                float d2 = __uint_as_float(r[h + 2]);
                float d3 = __uint_as_float(r[h + 3]);
                if (RELU == 2) {
                  d0 = fmaxf(d0, 0.f); d1 = fmaxf(d1, 0.f); d2 = fmaxf(d2, 0.f);
                  d3 = fmaxf(d3, 0.f);
                }
                acc01 = fma2(pack2(w4.x, w4.y), pack2(d0, d1), acc01);
                acc23 = fma2(pack2(w4.z, w4.w), pack2(d2, d3), acc23);
              }
              if ((c0 + 16) % C::HI == 0) {  // the query's last chunk: finish and store
                float a0, a1, a2, a3;
                unpack2(acc01, a0, a1);
                unpack2(acc23, a2, a3);
                float v = ((a0 + a1) + (a2 + a3)) * a.scale;
                if (RELU == 1) v = fmaxf(v, 0.f);
                const size_t row = (size_t)it.b * a.S + s;
                if constexpr (FILTER) {
                  // candidates of this query among the warp's 32 keys: one atomic per warp,
                  // the writes deferred to this query's next tile
                  Pending& p = pend[(cc * 16) / C::HI];  // compile-time slot
                  flush(p);
                  const uint32_t key = order_key(v);
                  const bool keep =
                      t < a.T && t <= s + a.q_off && key >= tau_q[(cc * 16) / C::HI];
                  p.bal = __ballot_sync(0xffffffffu, keep);
                  p.key = key;
                  p.t = t;
                  p.off = row * (size_t)a.cand_cap;
                  p.base = 0;
                  if (p.bal && lane == 0) p.base = atomicAdd(a.cand_cnt + row, __popc(p.bal));
                } else if (t < a.T) {
                  a.scores[row * a.ldT + tcol] = (t <= s + a.q_off) ? v : ninf;
                }
                acc01 = acc23 = pack2(0.f, 0.f);
              }
            }
          }
          if (cc + 1 < NCH) {
            if constexpr (NBUF == 1) tmem_ld16(t_lane + ab * C::ACC_COLS + col0 + (cc + 1) * 16, rb[0]);
            tmem_wait_ld();
          }
        }
        ++ci;
      }
    }
    if constexpr (FILTER) {
#pragma unroll
      for (int q = 0; q < QW; ++q) flush(pend[q]);
    }
