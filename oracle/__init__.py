"""Plain float64 CPU oracle for the TurboQuant hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
anything in this package.  The product path (the CUDA library and its Python
binding) never calls it and fails loudly when its compiled extension is missing.

The oracle shares no code with the CUDA path: it implements every step from the
pages' description in numpy / scipy float64, in the pages' order and notation,
without blocking, fusion or reordering.  Where the pages leave a step open the
plainest reading is taken and named in the function's docstring.

Sources (cited by page and section in each function):
  [ZX]  zingnex.cn forum thread "TurboQuant：接近理论极限的KV缓存量化方案",
        sections "随机旋转与Beta分布" and "两阶段内积量化".
  [TQN] turboquant.net landing page ("为什么 TurboQuant 是 AI 领域的'核弹级'突破？"),
        sections "PolarQuant：极坐标变换 / 坐标分布公式", "伪代码实现步骤"
        (预计算 Lloyd-Max 质心, 生成随机旋转矩阵, Quant / DeQuant 函数, 集成到 Attention)
        and "潜在挑战与解决方案" (随机旋转开销, 残差 norm 存储).
  [ADM] admirer.cn news article on Google Research's TurboQuant, paragraphs on
        PolarQuant (random rotation, Beta coordinates, Lloyd-Max), QJL (1-bit sign
        sketch, unbiased inner products), the two-stage b-1 + 1 bit pipeline and the
        vector-search comparison (GloVe d=200, 1@k recall, indexing time).

Pins: every function is checked by ``tests/test_oracle_*.py`` against closed forms,
textbook tables, brute force or Monte-Carlo invariants (see those tests).  Parity
of the search recall figure is unpinned by the pages (their recall charts did not
survive extraction); the search oracle itself is pinned by brute force.
"""
from .rng import splitmix64, uniform01, gaussian_stream
from .params import (
    haar_rotation, beta_coordinate_density, beta_coordinate_cdf, lloyd_max,
    lloyd_max_beta, lloyd_max_gaussian, make_params,
)
from .quantize import quantize, dequantize, dequantize_qjl, fp16_round
from .estimate import (
    prepare_query, estimate_inner_products, decode_attention, search_topk, recall_at,
)

__all__ = [
    "splitmix64", "uniform01", "gaussian_stream", "haar_rotation",
    "beta_coordinate_density", "beta_coordinate_cdf", "lloyd_max", "lloyd_max_beta",
    "lloyd_max_gaussian", "make_params", "quantize", "dequantize", "dequantize_qjl", "fp16_round",
    "prepare_query", "estimate_inner_products", "decode_attention", "search_topk",
    "recall_at",
]
