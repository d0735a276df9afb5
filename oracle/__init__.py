"""CPU oracle for one early-skipping denoising step of a masked-diffusion transformer.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The product (the CUDA library and its Python binding) never imports,
links or calls it, and it shares no code with the product: the only common
module is ``synth``, which draws the seeded inputs and holds none of the
method's arithmetic.

The oracle is written for a reader checking it against the pages by eye:
float64 numpy, one function per step of the method, no blocking, fusion or
reordering. Values are rounded to the storage type ("f32" or "bf16") exactly
at the storage points listed in ``oracle.model`` and nowhere else.

Sources (web summaries of two papers; cited by title and section):

* "ES-dLLM: Efficient Inference for Diffusion Large Language Models by
  Early-Skipping", technical summary: section 1 (every iteration processes the
  whole sequence; only the most confident masked tokens are unmasked),
  section 2.A (importance score equation I_{l,i}, alpha = 0.5, d = hidden
  size), section 2.B (top-k with k = (1 - r_l)|S|, skipped tokens bypass the
  later layers, K/V/hidden-state caches updated in place by scatter for the
  selected tokens and reused for the skipped ones, periodic full refresh of
  the prompt or current block).
* "DyLLM: Efficient Diffusion LLM Inference via Saliency-based Token Selection
  and Partial Attention", technical summary: section 2.B.2 (salient rows of
  the attention matrix are recomputed exactly = partial attention of the
  selected queries over all keys and values).

Parity status of each function is listed in ``oracle.model``'s header.
"""
from .model import *  # noqa: F401,F403
