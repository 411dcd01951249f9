"""Oracle for the few-step Flash DiT hot path: a plain, slow fp64 CPU restatement.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
anything in this package.  The product path (the ``few_step_dit_b200`` package
and its CUDA library) never imports it, and this package never imports the
product: the two share no code, headers, tables or helpers.

Sources (web write-ups of arXiv 2609.15863, "LynnReal-Omni"):

* [tokendh] tokendh.com news article on LynnReal-Omni, sections
  "一个模型如何同时干七件事：原生多模态骨干网络" (backbone, token tags),
  "训练的核心难题：怎么让模型又快又准" (flow matching, dual clocks, Flash
  layer schedule and spatial token compression).
* [PaperDaily] longzhangge PaperDaily, "LynnReal Lab视频恢复与生成：统一多模态控制，
  Flash降至377毫秒", section 一 (input tags, control offset, dual clocks) and
  section 二 "Flash怎么把22帧压到377毫秒" (compression, residual broadcast),
  section 三 "长视频不是无限塞历史，而是保留“够用的记忆”" (chunked long video).
* [tokendh] section "长视频生成：怎么记住十分钟前发生的事" (boundary frame,
  bounded multi-stride history) and section "解码器瓶颈：被忽视的那一半时间"
  (the 26-layer lightweight decoder).
* [ananclaw explainer] papers.ananclaw.com explainer of 2609.15863, section 3.4
  "推理加速" (the Flash model's lightweight VAE decoder).

Modules: ``dit.py`` (block, compression, stack, flow-matching sampler),
``long_video.py`` (chunked generation with the bounded history; import it as
``oracle.long_video``), ``fp8.py`` (E4M3 block projections; ``oracle.fp8``)
and ``decoder.py`` (the lightweight decoder's forward; ``oracle.decoder``).

Every floating-point step runs in float64.  Where the pages leave a step open
the plainest reading is taken; each one is marked ``Reading:`` in the docstring.

Parity status per function: every public function is called by a named pin
(``tests/test_oracle_composition.py`` checks that none is missing).  The
pieces of ``dit.py`` are pinned in ``tests/test_oracle_pins.py``; its
composites (the timestep MLP, the output heads, the stack with the Flash
schedule and the sampler with its two clocks) in
``tests/test_oracle_composition.py``, by weights that reduce each one to a
closed form; ``long_video.py`` in ``tests/test_oracle_long_video.py``,
``fp8.py`` in ``tests/test_oracle_fp8.py`` and ``decoder.py`` in
``tests/test_oracle_decoder.py``.  Three conventions are definitions that no
page fixes (the weight init, the timestep MLP's layer sizes and activation,
which projections carry biases): the pins check the wiring the oracle gives
them, and the GPU path is compared against that definition.
"""

from .dit import *  # noqa: F401,F403
