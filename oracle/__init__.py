"""CPU oracle for SSM-layer decode -- TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 restatement of what the decode hot path computes, used to
check the CUDA library.  Nothing here is shared with the CUDA path (no kernels,
headers, helpers, tables or constant generators), and the product never imports
it: only tests/, the smoke check and the benchmark's CPU-baseline leg may.

  eager.c / eager.py  fp64 per-token eager recurrence (Mamba-2, Gated DeltaNet,
                      Kimi Delta Attention), OpenMP
  closed_form.py      brute-force unrolled closed forms (tiny inputs)
  ut_form.py          chunked (WY / UT) fold of the delta-rule layers
  prefill.py          chunked Mamba-2 prefill (outputs and the checkpoint after a prompt)
  replay.py           fp64 checkpoint + buffer formulation, and the single
                      low-precision-state eager comparator
  ring.py             integer model of counters, ring slots, flush, verify/commit
  quant.py            bf16 / per-row fp8 e4m3 quantiser emulation
"""
