"""Plain CPU oracle for GPTQ layer quantization.

TEST INFRASTRUCTURE ONLY. Nothing in the product package imports, calls or
links anything in this directory; only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` use it.  It shares
no code with the CUDA path: no kernels, headers, helpers or constants.

Every function restates, in float64 NumPy, a step that the source pages
describe; each cites the page and section it follows.  The pages are:

* "第5章 GPTQ 实战：如何把 Hugging Face 模型量化成 4-bit" (CSDN chapter 5),
  cited as [ch5 §5.1.x];
* "AutoGPTQ 官方示例全解析" (AutoGPTQ examples guide), cited as [examples §1.4];
* "gptq" skill card (skillsbot), cited as [skill card, 分组量化];
* "OLMo 仓库中的 AutoGPTQ 快速上手" (OLMo quick-start), cited as [OLMo §三].

Pins that tie each function to something other than itself live in
``tests/test_oracle_*.py``.  Functions without such a pin say
"parity unpinned" in their docstring.
"""

from .gptq_ref import *  # noqa: F401,F403
