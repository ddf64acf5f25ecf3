"""CPU oracle for packed-KV online-softmax attention.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
restatement of what the pages compute.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and its
``--impl reference`` arm) may import it.  The CUDA product path in ``sm_b200``
never imports, links or calls anything here, and nothing here imports
``sm_b200``; the two share no code.

Every function names the page and section it follows.  Pages:

* "KV分组打包：4-bit到底省了多少？" (huhohoo.com/docs/llm/kv-packed-groups) --
  the symmetric 4/8-bit group format, nibble packing, grouping axes, padding
  and cropping, the byte ledger table.
* "Block KV decoding: less workspace, more time"
  (huhohoo.com/en/docs/llm/kv-block-decode-cost) -- the m/z/u block merge,
  dense-vs-blocked tolerance, the workspace-array table.
* "注意力分塊：不保存完整分數矩陣，如何保持結果？"
  (huhohoo.com/zh-TW/docs/llm/tiled-online-softmax) -- why block averaging is
  wrong, the three running quantities, block length 7.
* "给长前缀列一张有单位的资源账本" (codingai-lec05.pages.dev, resource-ledger)
  -- softmax(QK^T/sqrt(d_k))V, GQA sharing, mask rules, the 17/3 example.

Parity status: every public function is pinned by ``tests/test_oracle_pins.py``
against values the pages print, closed forms, brute force or error bounds
(``rel_l2_error`` by closed forms); only the magnitudes of the pages' error
table are a soft band (their random inputs cannot be regenerated) -- that
band is "parity unpinned" at the value level.
"""

from .kvq_oracle import (  # noqa: F401
    PackedMatrix,
    QMAX,
    pair_nibbles,
    split_nibbles,
    quantize_groups,
    pack_k,
    pack_v,
    pack_matrix,
    unpack_matrix,
    unpack_rows,
    payload_bytes,
    fixed_array_bytes,
    attend_dense,
    attend_blocked,
    attend_blocked_packed,
    attend_bruteforce,
    merge_partials,
    partial_state,
    attend_gqa,
    attend_gqa_heads,
    attend_gqa_window,
    attend_gqa_causal,
    rel_l2_error,
)
