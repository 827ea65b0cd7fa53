"""CPU oracle for the latent-KV decode path: test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline and
reference legs may import this package.  The product path never does.
"""
