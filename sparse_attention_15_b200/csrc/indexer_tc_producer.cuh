// A fragment of index_scores_tc_kernel's body (indexer_tc.cu): the TMA producer role.  The kernel
// includes it twice, once under the register split (inside the branch of a warpgroup,
// after its setmaxnreg) and once in the flat role dispatch of the kernels without the
// split, so that ptxas sees the same code in each form; lambdas or helper functions
// changed its register allocation.
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      UnitIter it(cta);
      uint32_t ai = 0, bi = 0;
      bool ok = true;
      while (ok && it.next(a, C::NQ, ncta)) {
        const int bb = bi % C::NB;
        if (bi >= (uint32_t)C::NB && !mbar_wait(&b_empty[bb], ((bi / C::NB) - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&b_full[bb], C::B_BYTES);
        const int qrow = (it.b * a.S + it.qb * C::NQ) * C::HI;
#pragma unroll
        for (int kh = 0; kh < C::KH; ++kh)
          tma_load_2d(Bs + bb * C::B_BYTES + kh * C::B_SLICE, &qmap, kh * C::SLICE_ELEMS, qrow,
                      &b_full[bb]);
        ++bi;
        for (int kt = it.k0; kt < it.k1; ++kt) {
          const int st = ai % C::NA;
          if (ai >= (uint32_t)C::NA && !mbar_wait(&a_empty[st], ((ai / C::NA) - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&a_full[st], C::A_BYTES);
          const int krow = it.b * a.T + kt * a.kstride * kTileM;
#pragma unroll
          for (int kh = 0; kh < C::KH; ++kh)
            tma_load_2d(As + st * C::A_BYTES + kh * C::A_SLICE, &kmap, kh * C::SLICE_ELEMS, krow,
                        &a_full[st]);
          ++ai;
        }
      }
      // on the way out, let every copy this thread issued land
      for (uint32_t j = (ai > (uint32_t)C::NA ? ai - C::NA : 0); j < ai; ++j)
        drain_wait(&a_full[j % C::NA], (j / C::NA) & 1);
      for (uint32_t j = (bi > (uint32_t)C::NB ? bi - C::NB : 0); j < bi; ++j)
        drain_wait(&b_full[j % C::NB], (j / C::NB) & 1);
    }
