"""BigBird ITC block-sparse attention (forward and backward) for B200.

The compute path is the C-ABI library ``libbbattn.so`` built from ``csrc/``;
``binding`` marshals arguments to it.  Importing this package loads nothing:
the library is loaded on first use and a missing library raises.
"""
