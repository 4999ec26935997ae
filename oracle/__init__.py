"""Float64 CPU oracle for the token-routed MoE SwiGLU FFN layer (forward + backward).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or link
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and its ``--impl reference`` arm) use it.
It shares no code with the CUDA library: no kernels, headers, helpers, tables or
constant generators, and it imports nothing from the CUDA package.

Sources.  The method is described only in prose on five news pages about the
Olmo-core 3 release.  Citations name the page and the section on it:

* ``kongchang`` -- "Ai2 Olmo-core 3：MoE训练吞吐量提升2.7倍的秘诀"
  (kongchang.com/articles/ai2-olmo-core-3-...).  Sections: 容量税 (capacity
  tax), 专家池扩展的实测数据 (expert-pool scaling measurements),
  路由不只是模型问题，更是系统问题 (routing is a systems problem),
  吞吐量数字的边界条件 (boundary conditions of the throughput numbers),
  代价在哪里 (where the cost is).
* ``aizyradar`` -- "Olmo-core 3:开源 MoE 训练框架,吞吐提升到原来的 2.7 倍"
  (aizyradar.cn/technologies/olmo-core-3).  Sections 改了什么 (what changed),
  数字 (numbers).
* ``aikraft`` -- "Прорыв в масштабируемости и производительности"
  (aikraft.ru/news/introducing-olmo-core-3-...).  Section "Технические
  оптимизации: от MXFP8 до маршрутизации" (technical optimisations).
* ``bytechap`` -- "Olmo-core 3 mở rộng quy mô đào tạo mixture-of-experts lên
  hàng nghìn tỷ tham số" (bytechap.com/vi/blog/olmo-core-3-...).  Section
  "Cách thức hoạt động" (how it works).
* ``promptowy`` -- "Olmo-core 3: otwarty system do trenowania modeli MoE w
  skali biliona parametrów" (promptowy.com/olmo-core-3-...).

The pages give no formulas.  Every place where the oracle had to pick a reading
(softmax router without renormalisation, lowest index wins ties, SwiGLU experts,
the OCP floor rule for MXFP8 scales, capacity rounding) is stated in the
docstring of the function that makes the choice.

Parity status: every public function is pinned by tests under ``tests/`` that
check it against brute force, closed forms, library routines, hand-derived
fixtures or finite differences (see ``tests/test_oracle_*.py``).
"""

from . import moe_ep_ref, moe_ref, mxfp8_ref  # noqa: F401
