"""Plain fp64 CPU oracle for FAVOR+ (Performer positive orthogonal random-feature attention).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or link this package:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use it. It
shares no code with the CUDA library (``linear_attention_positive_b200``) and imports nothing
from it.

Sources (the method is defined on these pages; citations name the page and the place on it):

* "Fast Attention Via Positive Orthogonal Random Features" (codewithpapers.app/method/favor),
  the FA-part equations: kernel attention A(i,j)=K(q_i,k_j), the random-feature identity
  K(x,y)=E[phi(x)^T phi(y)], the bidirectional output D^-1(Q'((K')^T V)) and the normaliser
  D = diag(Q'((K')^T 1_L)).
* "Rethinking Attention with Performers" (arXiv 2009.14794) abstract and the third-party summary
  page (aipaper.jasonlin.tech, "Key contributions" / "Limitations"): positive orthogonal random
  features, unbiasedness, low variance, orthogonal blocks with at most d rows.
* "Random Features for Efficient Attention Approximation" (Cambridge thesis record, abstract):
  masked (causal) self-attention.

The positive map phi(x) = exp(Wx - |x|^2/2)/sqrt(m), the block-orthogonal draw with chi(d) row
norms, the causal prefix-sum form and the backward pass are not printed on the pages; the
readings taken for them are listed in each module's docstring.

Modules
-------
``philox``   Philox4x64-10 counter-based generator (Salmon et al., SC'11).
``features`` Gaussian draws and the block-orthogonal random feature matrix W.
``favor``    phi, bidirectional / causal forward, backward, the single-token causal step,
             brute-force definitions, softmax.
``kernels``  generalised attention (ReLU features) and the trigonometric softmax features.

Every function here is pinned by ``tests/test_oracle_*.py`` against something other than itself
(a library routine, brute force on the explicit L x L matrix, closed forms, Monte-Carlo bounds,
invariants, finite differences). No function is "parity unpinned".
"""

from . import philox, features, favor, kernels  # noqa: F401
