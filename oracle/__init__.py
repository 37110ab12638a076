"""CPU fp64 oracle for blockwise / ring softmax attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or call anything in this package.
The CUDA library never links, imports or calls it, and nothing here imports the
CUDA library: the two share no code.  The only thing both sides consume is the
seeded input generator, which lives in its own module and holds none of the
method's arithmetic.

Sources (web pages, cited by title and section):

* [GC]  blog.gitcode.com, "分布式注意力机制突破：长序列处理的全景技术架构与实践指南"
        (distributed attention overview): §2.2 phase 3 (pairwise LSE merge),
        §3.4 (M-way merge through per-device (m_i, s_i)).
* [VR]  vibe-research.pages.dev, "架构层解决方案 - Sparse Attention与Ring Attention":
        "Ring Attention" section, the blockwise softmax identity and the ring
        sequence diagram (KV blocks rotate, each node accumulates); "MQA与GQA"
        section (query-head groups sharing one K/V head).
* [KK]  git.kang-kang.com, "注意力机制演进": timeline (Striped Attention),
        "FlashAttention" data-flow figure, "Ring Attention" figure.
* [FA]  intelliparadigm.com, "深度学习注意力机制优化与FlashAttention实践":
        §2.1 (standard attention), §2.2 (memory arithmetic), §3.3 and §4.1
        (the backward pass recomputes the weights), §4.2 (online softmax
        pseudocode), §5.1 (fp32 for log/exp, causal mask).
* [MO]  intelliparadigm.com, "Mosaic多轴注意力分片：突破Transformer长序列处理瓶颈":
        §2.1 (softmax(QK^T/sqrt(d))V, 150k-token memory), §2.2 (tabular
        tensors), §3.2 (ring steps: GPU 0 receives K3,V3 from GPU 3).

Every function in ``fp64.py`` is pinned by ``tests/test_oracle_pins.py``
against closed forms, hand-derived worked examples (``tests/golden``), brute
force in pure Python, invariants, and a library routine on special cases.
No function is "parity unpinned".
"""

from .fp64 import (  # noqa: F401
    NEG_INF,
    token_positions,
    allowed_mask,
    probabilities,
    attention,
    attention_rows,
    online_softmax_attention,
    lse_pair,
    merge_pair,
    merge_many,
    ring_attention,
    score_matrix_bytes,
    kv_head,
    attention_backward,
)
from .sampling import sample_rows  # noqa: F401
