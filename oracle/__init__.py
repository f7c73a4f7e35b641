"""CPU oracle for the NVFP4 / MXFP8 hot path -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package.  The product path never does.
"""
