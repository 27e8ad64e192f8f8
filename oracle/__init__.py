"""Double-precision CPU oracle for the DSpark hot path.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT: only tests/, the package
smoke check (__graft_entry__.smoke) and bench.py's CPU-baseline leg may
import this package.
"""
