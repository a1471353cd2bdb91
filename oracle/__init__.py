"""FP64 CPU oracle for exact route-set Query Sparse Attention (QSA).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its Python binding) never imports, calls or links it,
and this package imports nothing from the product path.

Every function here is a plain, slow, obviously correct restatement of what the
documentation pages define; see ``qsa_oracle`` for the citations.
"""

from .qsa_oracle import (  # noqa: F401
    routes_to_membership,
    row_route_sets,
    forward_dense,
    backward_dense,
    forward_rows,
    backward_rows,
    backward_keys,
    route_rows_csr,
    key_quad_lists,
    key_tile_lists,
    query_union_lists,
)
