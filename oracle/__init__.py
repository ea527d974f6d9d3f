"""Oracle: plain, slow, obviously correct CPU implementation of causal prefill attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import, call, link or
execute anything in this package.  The product path (the C-ABI library and its Python
binding) never touches it, and this package never imports the product package.

Sources followed (the three web pages on Zyphra's ZYFA release):
  [ZYFA-pt] acheiumaia.com.br, news item "zyphra-zyfa-flashattention-fp8-para-amd-mi355x"
            (TL;DR; "Por que a atenção FP8 tem desempenho inferior no MI355X?";
            "Como o ZYFA funciona?")
  [ZYFA-mb] miraibroadcast.com, "Zyphra lança ZYFA e acelera GPUs AMD em até 1,76x IA"
            ("Como o motor de atenção FP8 da Zyphra funciona";
            "Precisão, estabilidade e efeito na prática")
  [ZYFA-fr] ai-daily-news.org, article "zyphra-zyfa-fp8-flashattention-amd-mi355x"
            ("L'essentiel en 30 secondes"; "Ce que couvrent les noyaux")

Modules
  attention  fp64 causal attention (the plain definition), full and sampled rows
  e4m3       OCP e4m3fn codec (decode, round-to-nearest-even saturating encode)
  hadamard   Sylvester-Hadamard rotation along the head dimension
  quantize   per-tensor e4m3 quantisation (+ optional rotation)
  leanp      bit-level lean-P / power-of-two block-scale emulator (plain C, via ctypes),
             and the exact-P ablation (exponential then e4m3 rounding)
  decode     fp64 decode attention over a paged KV cache (one query token per sequence)

Pins (what each function is checked against, in ``tests/test_oracle_*.py``):
  attention  brute force on tiny inputs, 2x2 hand-computed case, Q=0 prefix mean,
             rows of P sum to 1, O[0]=V[0], masked keys have zero influence,
             GQA == MHA with repeated K/V heads, shift invariance in K.
  e4m3       exhaustive against torch.float8_e4m3fn (all 256 codes, all midpoints,
             a dense fp32 sweep), saturation beyond 448.
  hadamard   H H^T = 128 I, recursive Sylvester structure, round trip, explicit matrix.
  quantize   codes and descale recomputed from the e4m3 value table by brute force.
  leanp      closed forms (s = max gives byte 8*(7+k)), Mitchell error bound,
             monotonicity, exact fma against rational arithmetic, and the end-to-end
             tile driver against fp64 attention within the FP8 tolerance; exact P:
             power-of-two closed forms, e4m3 rounding bound, driver pinned to the C one.
  decode     equals the last row of the (pinned) prefill oracle on the gathered
             sequence, page-permutation invariance, length 1 gives v_0, Q = 0 gives the
             mean of V, an empty sequence gives zeros.
"""
