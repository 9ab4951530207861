// A fragment of index_scores_tc_kernel's body (indexer_tc.cu): the MMA issuer role.  The kernel
// includes it twice, once under the register split (inside the branch of a warpgroup,
// after its setmaxnreg) and once in the flat role dispatch of the kernels without the
// split, so that ptxas sees the same code in each form; lambdas or helper functions
// changed its register allocation.
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc =
          C::ES == 2 ? idesc_bf16_f32(kTileM, C::N) : idesc_e4m3_f32(kTileM, C::N);
      UnitIter it(cta);
      uint32_t ai = 0, bi = 0, ci = 0;
      bool ok = true;
      while (ok && it.next(a, C::NQ, ncta)) {
        const int bb = bi % C::NB;
        if (!mbar_wait(&b_full[bb], (bi / C::NB) & 1)) { ok = false; break; }
        const uint32_t b_base = smem_u32(Bs + bb * C::B_BYTES);
        for (int kt = it.k0; kt < it.k1; ++kt) {
          const int st = ai % C::NA;
          if (!mbar_wait(&a_full[st], (ai / C::NA) & 1)) { ok = false; break; }
          const int ab = ci % C::NACC;
          if (ci >= (uint32_t)C::NACC &&
              !mbar_wait(&acc_empty[ab], ((ci / C::NACC) - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(As + st * C::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < C::ROW_BYTES / 32; ++kk) {
            const uint32_t off = (kk & 3) * 32;  // 32 B (16 bf16 / 32 e4m3) along the row
            const uint64_t adesc = sw128_kmajor_desc(a_base + (kk >> 2) * C::A_SLICE + off);
            const uint64_t bdesc = sw128_kmajor_desc(b_base + (kk >> 2) * C::B_SLICE + off);
            if constexpr (C::ES == 2)
              umma_f16_ss(tmem + ab * C::ACC_COLS, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
            else
              umma_f8f6f4_ss(tmem + ab * C::ACC_COLS, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&a_empty[st]);
          umma_commit(&acc_full[ab]);
          ++ai;
          ++ci;
        }
        if (!ok) break;
        umma_commit(&b_empty[bb]);
        ++bi;
      }
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
