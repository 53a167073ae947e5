"""CPU oracle for one DiffusionGemma denoising step — TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, float64 restatement of the method described on
the DiffusionGemma pages (the arXiv abstract page "DiffusionGemma 技术报告",
the popular-science article on laozijiushiniubi.cn whose §二 and §四 give the
model and sampler details, and the chatpaper.ai abstract).  It exists so the
CUDA library can be checked against it; nothing in the product path may import
it.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg use it.

It shares no code with the CUDA library.  Its only shared dependency is the
seeded input generator in ``synth/`` (weights and token ids are inputs).

A second, plain C++ implementation of the same round and of the causal
encoding (``dg_oracle.cpp``, double precision with plain loops, reached
through ``oracle.cpp``) shares no code with this one either; the tests run
both on the same seeded weights and inputs and require them to agree at
every decision point.

Parity status per function is recorded in each module's docstring; the one
part with no independent closed-form pin is the composition of the full
random-init model (``forward_layers`` over many layers): "parity unpinned"
beyond its pinned components, and cross-checked only by the C++ oracle.
"""

from .philox import philox4x32_10, uniform_token, gumbel_u  # noqa: F401
from .numerics import bf16_round, f32_round, bf16_bits_to_f64  # noqa: F401
from .model import (  # noqa: F401
    ModelConfig,
    Weights,
    KVCache,
    rmsnorm,
    rope,
    attention,
    moe_ffn,
    route,
    forward_layers,
)
from .sampler import (  # noqa: F401
    SamplerConfig,
    temperature,
    position_stats,
    gumbel_sample,
    lock_mask,
    stop_flag,
    expected_embedding,
)
from .decode import (  # noqa: F401
    CanvasState,
    StepOutput,
    init_canvas,
    encode_context,
    denoise_step,
    decode_block,
)
