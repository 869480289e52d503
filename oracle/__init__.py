"""Plain CPU reference (the oracle) for the routed-expert MoE layer on 4-bit
block-scaled weights.

TEST INFRASTRUCTURE ONLY. Nothing in the library may import, call or link
anything here: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. The
oracle shares no code with the CUDA path; the only module both sides use is
``synth`` (seeded input generation, none of the method's arithmetic).

Everything is numpy in float64 unless a passage of the pages fixes another
precision; the NVFP4 scale computation follows the float32 operation order
spelled out in ``oracle.formats`` because it decides integer codes.

Sources, cited by page title and section:
  [XFP]  "XFP：质量地板驱动的自适应码本量化——3.4 位在双卡工作站跑通 397B MoE"
         (pinghaoyang.com.cn/aigc/posts/xfp): sections 路线二 (hardware
         formats NVFP4 / MXFP4), 路线一 (the 49-sigma worked example),
         V2 (codebook + outlier triples), 离群值提取 (outlier extraction),
         Lloyd 迭代 (Lloyd iterations), 子字节打包 (sub-byte packing),
         V2a (shared library, effective bits).
  [GATE] "The gate that missed by 0.0202 pp" (jinnpan.com,
         glm53-mxfp4-mi355x): sections "A file is a census; a decode step
         is a sample" (active bytes, top-8 of 288 / 256 experts) and
         "A fused tensor with two dtypes in it" (two values per byte,
         fused expert buffer).
  [CARD] "GLM-5.3-Flash-MXFP4" model card (aimarketly): section
         "Verification compute and EAGLE" (experts keep the SwiGLU gate
         and its clamp).
  [TF]   TensorFold pull request #1050: checked shape arithmetic with
         named refusals (EmptyShape, ShapeOverflow); W4A16_NVFP4 packing
         with a global scale.

Parity pins (tests/test_oracle_*.py) tie every function here to facts the
pages or mathematics fix; see each module's docstring for which.
"""
from . import formats, codebook, routing, moe, v2a  # noqa: F401
