"""CPU oracle for DeepSeek-V4 hybrid compressed attention (CSA / HCA).

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, fp64 numpy
restatement of what the hot path computes, written from the pages' statement
of the method.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library never imports, links or calls anything here, and nothing
here imports the CUDA package; the two share only the seeded input generator
``synth``.

Sources (cited by page title and section throughout):
  [deep-read]  "DeepSeek-V4 深读：百万 Token 不是窗口数字，而是一整套系统契约"
               (ricardokevins.github.io) - sections "CSA：4× 压缩之后再 top-k"
               (equation C_i^comp), "HCA：128× 压缩后保留 dense 全局视野",
               "其他稳定性细节" (RMSNorm, partial RoPE, output inverse rotation,
               attention sink, FP8/BF16 KV, FP4 indexer), the model-spec table
               ("模型规格": heads, head dim, top-k, RoPE theta), "FP4 QAT、可恢复
               rollout 与百万 Token RL" (MXFP4 indexer QK path).
  [summary]    "DeepSeek-V4: Towards Highly Efficient Million-Token Context
               Intelligence (arXiv 2026)" (awesome-system-papers.pages.dev) -
               section "核心方法 / Hybrid CSA + HCA Attention".
  [news]       "AI深一度 第15期|DeepSeek V4" (yeyulingfeng.com) - section
               "一、CSA与HCA" (softmax-gated pooling with a learnable position
               bias) and "二、FP4闪电索引与混合精度KV缓存".
  [notes]      "拆解 DeepSeekv4" (daixd5520.github.io) - sections "CSA" (half
               overlapping windows), "HCA", "细节" (per-head Q RMSNorm and
               shared-KV RMSNorm, RoPE on the last 64 dims, sink exp(z'_h) in
               the softmax denominator, 128-token window).
  Number formats: OCP 8-bit Floating Point Specification (OFP8) rev 1.0
  (E4M3) and OCP Microscaling Formats (MX) Specification v1.0 (E2M1, E8M0).

Where the pages are silent, the oracle takes one reading (R1..R16) and names
it at the point of use.  Every function is pinned by tests under
``tests/test_oracle_*.py`` against invariants, closed forms, library routines
or brute force; none is "parity unpinned".
"""
