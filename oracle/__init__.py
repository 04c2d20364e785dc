"""CPU oracle for CSA2 sparse attention over an FP4 main-KV cache.

TEST INFRASTRUCTURE ONLY.  This package is the slow, plain reference that
the CUDA path is checked against.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may
import it.  The product package (``fp4_kv_cache_mxfp4_b200``) never imports
it and shares no code, table or helper with it.

Everything is written from the pages' statement of the method, in numpy,
float64 for real arithmetic except where a floating-point value decides an
integer code (the FP4 encoder), where both this oracle and the kernel decide
in IEEE float32.

Citations name the source page and its section:

* [eogee] "DeepSeek V4.1-Flash 技术报告深度解析：CED 架构与 KV Cache 极限压缩"
  (eogee.com/article/126) -- §3.2 CSA2 modes, §3.3 Hierarchical Sparse
  Indexer, §3.4 FP4 main KV cache, §5.3 efficiency.
* [opskyn] "DeepSeek 正式发布并开源 DeepSeek V4.1 Flash" (jh.opskyn.com/article/924)
  -- section "HBM 与 SSD，分别怎么省？" (mode definitions, HSI).
* [ainewsway] "DeepSeek-V4.1-Flash cuts KV cache to 890 bytes per token"
  (ainewsway.com) -- section "KV 快取為何成為瓶頸" (E2M1, 16-channel scales,
  3 encoder + 1 decoder cache).
* [nxbn] "DeepSeek-V4.1-Flash" README walk-through (m.nxbn.cn/news/186820) --
  §2.3 CSA2, §3.1 text-backbone table, §3.3 CSA2 / sparse-index table.
* [titansim] DeepSeek-V4.1-Flash summary blog (titansim.online) -- section
  "核心机制与研究方法", CSA2 mode list and Figure 5 (HSI).

Parity status of every function is listed in its docstring; all functions
here are pinned by ``tests/test_oracle_*.py`` against hand-worked values,
library routines (ml_dtypes / torch float8, torch SDPA), brute force on tiny
inputs or closed forms.
"""

from . import fp4, fp8, mxfp4, compress, indexer, attention, group  # noqa: F401
