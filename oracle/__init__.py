"""fp64 CPU attention oracle -- test infrastructure only (tests, smoke check, CPU baseline)."""
