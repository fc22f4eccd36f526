"""CPU oracle for the MoT world-action-model forward (TEST INFRASTRUCTURE).

This package is the plain, slow, obviously-correct statement of what the
CUDA library computes.  It exists to check the library, never to stand in
for it: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg (``--impl reference`` and the ``cpu_baseline`` field) may
import it.  The product path (``mot_dit_b200``) never imports it and has no
CPU fallback.

The oracle shares no code with the CUDA path: it has its own configuration
presets, its own parameter generator (the counter-based splitmix64 /
Box-Muller rule, written here in numpy) and its own forward pass in float64.
The only module both sides use is ``synthetic`` (seeded chunk inputs).

Sources.  All formulas follow the pages on "RealtimeWAM: One-Step Asynchronous
World Action Models" (paper.rainbus.top summary, sections 前置知识 / 核心方法 /
方法步骤详情; tokendh.com article, CEWP section) and the Flash-WAM close reading
(auto-driving-blog, sections 概念 / 方法 / 数据与训练流程).  Where the pages
leave a step open the reading taken is named in the function's docstring.

Modules:
    config  -- model shapes and the five synthetic presets
    params  -- seeded parameter generation (N(0, 0.02) weights, unit gains)
    model   -- float64 forward: video expert, action expert, Euler / endpoints
    tacd    -- TACD training targets, forward only: teacher K-step rollout,
               interval-average velocity, student / EMA endpoints, L_TA, L_CD
    multistep -- chunk with a multi-step video expert: N_v Euler steps of the
               video latents, the action expert on the last forward's K/V
"""
from .config import WamConfig, preset  # noqa: F401
from .params import generate_params, param_specs  # noqa: F401
from . import model  # noqa: F401
