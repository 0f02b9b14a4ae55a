"""CPU oracle for the group-wise MinMax quantizer and weight-only linear.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the product package.
"""
