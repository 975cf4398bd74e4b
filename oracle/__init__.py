"""Float64 CPU oracle for the gated delta rule.  Test infrastructure only:
the product path never imports this package."""
